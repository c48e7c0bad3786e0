"""Guard bytes around the caller-owned page pools.

Each of the four pools sits inside a larger device buffer whose margins (4 KiB
on each side) hold a fixed pattern.  Appends, decodes (tensor-core and
CUDA-core paths) and a prefill then run on the pools; after each call the
margins must be unchanged, and every result must still match the oracle.  A
write past either end of a pool shows up as a changed margin.
"""
import numpy as np
import pytest
import torch

import oracle as O
from harness import gen

from _cases import bf16_tensor, check_attention, make_ctx, oracle_cache, skv, upload

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


class GuardedCache:
    """The four pools of a cache, each in the middle of a guarded buffer."""

    def __init__(self, S, cfg, n_pages):
        self.sizes = S.starkv_cache_layout(cfg, n_pages)
        self.n_pages = n_pages
        self.bufs, ptrs = {}, []
        for name in ("k_codes", "v_codes", "k_meta", "v_meta"):
            n = self.sizes[name + "_bytes"]
            buf = torch.full((n + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
            self.bufs[name] = buf
            setattr(self, name, buf[GUARD:GUARD + n])
            ptrs.append(buf.data_ptr() + GUARD)
        self.struct = S.starkv_cache(*ptrs, n_pages)

    def damaged(self):
        bad = []
        for name, buf in self.bufs.items():
            n = self.sizes[name + "_bytes"]
            if not bool((buf[:GUARD] == PATTERN).all()) or not bool((buf[GUARD + n:] == PATTERN).all()):
                bad.append(name)
        return bad


def _i32(x):
    return torch.tensor(np.asarray(x, np.int32)).cuda()


@pytest.mark.parametrize("path", ["tensor-core", "cuda-core"])
def test_page_pool_margins_survive_append_decode_prefill(monkeypatch, path):
    if path == "cuda-core":
        monkeypatch.setenv("STARKV_DECODE_PATH", "simt")
    S = skv()
    w = gen.workload("longchat7b_decode_b16_t4096")
    lens, caps = [33, 300], [64, 330]
    kv, f = make_ctx(w, max_position=400)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, lens, extra_pages=2, caps=caps)
        gc = GuardedCache(S, kv.cfg, n_pages)
        upload(gc, oc)
        btd = torch.from_numpy(bt).cuda()
        q = gen.make_queries(2, w.H, w.d_h, name="q_step", sub=900)

        out = kv.decode(gc, bf16_tensor(q), btd, _i32(lens))
        check_attention(out.float().cpu().numpy(), O.decode(oc, q, f.B_k, f.B_v, bt, lens), f"{path} decode")
        assert gc.damaged() == []

        # two new tokens per sequence, then the grown context
        X = gen.make_hidden(4, w.hidden, name="X_step", sub=900)
        sl = np.concatenate([gen.slots_for(bt, b, [L, L + 1]) for b, L in enumerate(lens)])
        S.starkv_append(kv.ctx, gc.struct, bf16_tensor(X), torch.from_numpy(sl).cuda())
        O.append(oc, X, f.A_k, f.A_v, sl)
        assert gc.damaged() == []
        lens2 = [L + 2 for L in lens]
        out = kv.decode(gc, bf16_tensor(q), btd, _i32(lens2))
        check_attention(out.float().cpu().numpy(), O.decode(oc, q, f.B_k, f.B_v, bt, lens2),
                        f"{path} decode after append")
        assert gc.damaged() == []

        # a 20-token chunk per sequence, appended, then attended causally
        chunks = [20, 20]
        totals = [L + c for L, c in zip(lens2, chunks)]
        Xc = gen.make_hidden(sum(chunks), w.hidden, name="X_chunk", sub=900)
        slc = np.concatenate([gen.slots_for(bt, b, np.arange(L, L + c))
                              for b, (L, c) in enumerate(zip(lens2, chunks))])
        S.starkv_append(kv.ctx, gc.struct, bf16_tensor(Xc), torch.from_numpy(slc).cuda())
        O.append(oc, Xc, f.A_k, f.A_v, slc)
        cu = np.array([0, chunks[0], sum(chunks)], np.int32)
        qc = gen.make_queries(sum(chunks), w.H, w.d_h, name="q_chunk", sub=900)
        out = kv.prefill(gc, bf16_tensor(qc), torch.from_numpy(cu).cuda(), btd, _i32(totals), max(chunks))
        check_attention(out.float().cpu().numpy(), O.prefill(oc, qc, cu, f.B_k, f.B_v, bt, totals),
                        f"{path} prefill")
        assert gc.damaged() == []
        assert kv.status() == 0
    finally:
        kv.close()
