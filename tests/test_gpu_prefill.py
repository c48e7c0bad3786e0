"""GPU parity of starkv_prefill_attn (causal chunk attention) against the oracle.

The existing context comes from an oracle-written cache; the chunk's own
tokens are appended by each side with its own arithmetic from the same hidden
states, then every chunk query attends causally."""
import numpy as np
import pytest
import torch

import oracle as O
from harness import gen

from _cases import bf16_tensor, check_attention, make_ctx, oracle_cache, skv, upload

pytestmark = pytest.mark.gpu


def run_prefill(w, existing, chunks, seed=0, select=None):
    S = skv()
    totals = [e + c for e, c in zip(existing, chunks)]
    kv, f = make_ctx(w, seed, max_position=max(totals) + 16)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, existing, seed, extra_pages=2, caps=totals)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        cu = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
        Xs, slots = [], []
        for b, (e, c) in enumerate(zip(existing, chunks)):
            Xs.append(gen.make_hidden(c, w.hidden, seed, name="X_chunk", sub=b))
            slots.append(gen.slots_for(bt, b, np.arange(e, e + c)))
        X = np.concatenate(Xs)
        sl = np.concatenate(slots)
        S.starkv_append(kv.ctx, lc.struct, bf16_tensor(X), torch.from_numpy(sl).cuda())
        O.append(oc, X, f.A_k, f.A_v, sl)
        q = gen.make_queries(int(cu[-1]), w.H, w.d_h, seed, name="q_chunk")
        out = kv.prefill(lc, bf16_tensor(q), torch.from_numpy(cu).cuda(), torch.from_numpy(bt).cuda(),
                         torch.tensor(np.asarray(totals, np.int32)).cuda(), max(chunks))
        st = kv.status()
        ref = O.prefill(oc, q, cu, f.B_k, f.B_v, bt, totals, select=select)
        return out.float().cpu().numpy(), ref, st
    finally:
        kv.close()


def test_tiny_prefill():
    w = gen.workload(0)
    got, ref, st = run_prefill(w, [40, 0, 100], [9, 20, 37])
    assert st == 0
    check_attention(got, ref, "tiny prefill")


def test_tiny_prefill_cuda_core_path(monkeypatch):
    monkeypatch.setenv("STARKV_PREFILL_PATH", "simt")
    w = gen.workload(0)
    got, ref, st = run_prefill(w, [40, 0, 100], [9, 20, 37])
    assert st == 0
    check_attention(got, ref, "tiny prefill, CUDA-core path")


def test_prefill_several_query_and_key_tiles():
    # query tiles of 128 with a ragged last one, key tiles that straddle the
    # chunk boundary, a sequence that is all chunk (no earlier context)
    w = gen.workload(0)
    got, ref, st = run_prefill(w, [700, 0, 129], [300, 257, 128])
    assert st == 0
    check_attention(got, ref, "tiny prefill, several tiles")


def test_longchat_shapes_prefill_more_tiles():
    w = gen.workload(4)
    sel = {0: list(range(0, 260, 7)), 1: list(range(0, 131, 5))}
    got, ref, st = run_prefill(w, [1000, 0], [260, 131], select=sel)
    assert st == 0
    check_attention(got, ref, "longchat prefill, several tiles (sampled)")


def test_gqa_prefill_more_tiles():
    w = gen.workload(3)
    sel = {0: list(range(0, 200, 3))}
    got, ref, st = run_prefill(w, [383], [200], select=sel)
    assert st == 0
    check_attention(got, ref, "gqa prefill, several tiles (sampled)")


def test_prefill_bad_query_span_sets_status_and_zero_rows():
    S = skv()
    w = gen.workload(0)
    kv, f = make_ctx(w, max_position=256)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, [50], extra_pages=1)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        q = bf16_tensor(gen.make_queries(8, w.H, w.d_h))
        cu = torch.tensor([0, 8], dtype=torch.int32, device="cuda")
        sl = torch.tensor([5], dtype=torch.int32, device="cuda")         # 8 queries but only 5 positions
        out = torch.full_like(q, float("nan"))
        S.starkv_prefill_attn(kv.ctx, lc.struct, q, cu, torch.from_numpy(bt).cuda(), sl, 8, out,
                              kv.workspace(S.OP_PREFILL, 1, bt.shape[1], 8))
        assert kv.status() & S.DEV_BAD_QUERY_SPAN
        assert torch.all(out.float() == 0)
    finally:
        kv.close()


def test_longchat_shapes_prefill_small():
    w = gen.workload(4)
    got, ref, st = run_prefill(w, [300, 17], [64, 33])
    assert st == 0
    check_attention(got, ref, "longchat prefill small")


def test_gqa_prefill_small():
    w = gen.workload(3)
    got, ref, st = run_prefill(w, [128, 5], [50, 16])
    assert st == 0
    check_attention(got, ref, "gqa prefill small")


@pytest.mark.slow
def test_longchat_prefill_full_size_sampled():
    w = gen.workload(4)
    sel = {0: [0, 1, 1000, 2047], 3: [5, 2046]}
    got, ref, st = run_prefill(w, [w.ctx] * w.batch, [w.chunk] * w.batch, select=sel)
    assert st == 0
    check_attention(got, ref, "longchat prefill b4 t30720 c2048 (sampled)")
