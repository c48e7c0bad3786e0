"""Ragged key ranks: a learned rank per KV head ([Review] section 3 and its
figure of learned rank profiles; the checkpoint card caps the key rank at
max_rank_k = 64).  A synthetic profile of 16..64 per head through the layout,
the per-head quantiser, append, decode and prefill, against the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from harness import gen

from _cases import bf16_tensor, check_attention, download, make_ctx, oracle_cache, skv, upload

pytestmark = pytest.mark.gpu

PROFILES = {
    "llama3gqa": (3, (64, 48, 32, 16, 64, 32, 48, 16)),
    "tiny": (0, (16, 16, 16, 16)),
}


def _w(name, **kw):
    i, ranks = PROFILES[name]
    w = gen.workload(i)
    return gen.shrink(w, key_ranks=ranks, r_k=max(ranks), **kw)


def _longchat_profile():
    w = gen.workload(1)
    ranks = tuple([32, 16, 32, 32, 16, 32, 32, 32] * 4)
    return gen.shrink(w, key_ranks=ranks, r_k=32)


def test_ragged_layout_matches_oracle():
    S = skv()
    for w in (_w("llama3gqa"), _longchat_profile()):
        cfg = O.config_of(w)
        sz = S.starkv_cache_layout(S.make_config(w.H, w.h_kv, w.d_h, w.hidden, w.r_k, w.R, 64, w.top_fraction,
                                                 w.rope_base, 0, w.key_ranks), 5)
        want = O.layout_sizes(cfg, 5)
        assert (sz["k_codes_bytes"], sz["k_meta_bytes"], sz["v_codes_bytes"], sz["v_meta_bytes"]) == \
            (want["k_codes"], want["k_meta"], want["v_codes"], want["v_meta"])
        assert sz["key_page_bytes"] == cfg.key_layout()[1]


def test_ragged_rank_table_is_checked():
    S = skv()
    w = gen.workload(3)
    for ranks, code in (((64, 48, 32, 16, 64, 32, 48, 8), S.ERR_UNSUPPORTED_SHAPE),    # not a multiple of 16
                        ((48,) * 8, S.ERR_INVALID_ARG)):                                 # rank_k 64 != max 48
        with pytest.raises(S.StarKVError) as e:
            S.starkv_cache_layout(S.make_config(w.H, w.h_kv, w.d_h, w.hidden, 64, w.R, 64, 0.25, w.rope_base, 0,
                                                ranks), 1)
        assert e.value.code == code


def test_ragged_quantize_pack_per_head_bit_exact():
    S = skv()
    w = _w("llama3gqa")
    kv, f = make_ctx(w, max_position=64)
    try:
        cfg = O.config_of(w)
        for h in range(w.h_kv):
            lat = cfg.key_head(h)
            rng = np.random.default_rng(h)
            n = 21
            z = (rng.standard_normal((n, lat.r)) * rng.uniform(0.1, 9, (n, 1))).astype(np.float32)
            pages = 2
            codes = torch.zeros(pages * lat.region_bytes, dtype=torch.uint8, device="cuda")
            meta = torch.zeros(pages * lat.n_groups * 16, dtype=torch.int32, device="cuda")
            S.starkv_quantize_pack(kv.ctx, S.LATENT_KEY_HEAD(h), torch.from_numpy(z).cuda(), codes, meta)
            want_c, want_m = O.quantize_pack_region(z, lat)
            np.testing.assert_array_equal(codes.cpu().numpy().reshape(pages, -1), want_c)
            np.testing.assert_array_equal(meta.cpu().numpy().view(np.uint32).reshape(want_m.shape), want_m)
        assert kv.status() == 0
    finally:
        kv.close()


@pytest.mark.parametrize("n", [7, 200])
def test_ragged_append_bit_exact_on_exported_latents(n):
    S = skv()
    w = _w("llama3gqa", ctx=64)
    kv, f = make_ctx(w, max_position=n + 64)
    try:
        cfg = O.config_of(w)
        bt, n_pages = gen.make_block_table([n + 3], seed=2)
        slots = gen.slots_for(bt, 0, np.arange(3, 3 + n))
        X = gen.make_hidden(n, w.hidden, seed=5)
        lc = kv.new_cache(n_pages)
        kc = sum(w.key_ranks)
        lat = torch.zeros((n, kc + w.R), dtype=torch.float32, device="cuda")
        S.starkv_append(kv.ctx, lc.struct, bf16_tensor(X), torch.from_numpy(slots).cuda(), lat)
        assert kv.status() == 0
        zl = lat.cpu().numpy()
        oc = O.new_cache(cfg, n_pages)
        O.write_latents(oc, slots, O.pad_key_latents(cfg, zl[:, :kc]), zl[:, kc:])
        got = download(lc, oc)
        for name in ("k_codes", "v_codes", "k_meta", "v_meta"):
            np.testing.assert_array_equal(getattr(got, name), getattr(oc, name), err_msg=name)
        ref = np.concatenate([O.project(X, f.A_k), O.project(X, f.A_v)], axis=1)
        bound = 1e-5 * (np.abs(X).astype(np.float64) @ np.abs(np.concatenate([f.A_k, f.A_v], 1))) + 1e-30
        assert np.all(np.abs(zl - ref) <= bound)
    finally:
        kv.close()


@pytest.mark.parametrize("which", ["llama3gqa", "longchat", "tiny"])
def test_ragged_decode(which):
    w = _longchat_profile() if which == "longchat" else _w(which)
    lens = [700, 1300, 33] if which != "tiny" else [256, 17]
    kv, f = make_ctx(w, max_position=max(lens) + 16)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, lens, extra_pages=1)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        qn = gen.make_queries(len(lens), w.H, w.d_h)
        out = kv.decode(lc, bf16_tensor(qn), torch.from_numpy(bt).cuda(), torch.tensor(np.asarray(lens, np.int32)).cuda())
        assert kv.status() == 0
        ref = O.decode(oc, qn, O.pad_key_factor(cfg, f.B_k), f.B_v, bt, lens)
        check_attention(out.float().cpu().numpy(), ref, f"ragged decode ({which})")
    finally:
        kv.close()


def test_ragged_append_then_prefill():
    S = skv()
    w = _w("llama3gqa")
    existing, chunks = [260, 0], [90, 40]
    totals = [e + c for e, c in zip(existing, chunks)]
    kv, f = make_ctx(w, max_position=max(totals) + 16)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, existing, extra_pages=2, caps=totals)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        cu = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
        X = np.concatenate([gen.make_hidden(c, w.hidden, name="X_chunk", sub=b) for b, c in enumerate(chunks)])
        sl = np.concatenate([gen.slots_for(bt, b, np.arange(e, e + c)) for b, (e, c) in enumerate(zip(existing, chunks))])
        S.starkv_append(kv.ctx, lc.struct, bf16_tensor(X), torch.from_numpy(sl).cuda())
        O.append(oc, X, f.A_k, f.A_v, sl)
        q = gen.make_queries(int(cu[-1]), w.H, w.d_h, name="q_chunk")
        sel = {0: list(range(0, 90, 7)), 1: list(range(0, 40, 5))}
        out = kv.prefill(lc, bf16_tensor(q), torch.from_numpy(cu).cuda(), torch.from_numpy(bt).cuda(),
                         torch.tensor(np.asarray(totals, np.int32)).cuda(), max(chunks))
        assert kv.status() == 0
        check_attention(out.float().cpu().numpy(),
                        O.prefill(oc, q, cu, O.pad_key_factor(cfg, f.B_k), f.B_v, bt, totals, select=sel),
                        "ragged prefill")
    finally:
        kv.close()
