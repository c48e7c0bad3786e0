"""Pins of the oracle's attention path (CPU only).

Independent references: the transformers Llama RoPE helper, torch's
scaled-dot-product attention in fp64 on fully materialised keys/values,
dense attention with W_k = A_k B_k / W_v = A_v B_v, the softmax partition
identity, and closed-form special cases.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F
from transformers.models.llama.modeling_llama import apply_rotary_pos_emb

import oracle as O
from harness import gen


def hf_rope(x, pos, base):
    """RoPE via transformers' Llama helper (rotate_half convention), fp64."""
    x = torch.as_tensor(np.asarray(x, np.float64))          # [n, d]
    d = x.shape[-1]
    inv = 1.0 / (base ** (torch.arange(0, d, 2, dtype=torch.float64) / d))
    fr = torch.as_tensor(np.asarray(pos, np.float64))[:, None] * inv[None]
    emb = torch.cat([fr, fr], -1)
    cos, sin = emb.cos()[None], emb.sin()[None]           # [1, n, d]
    q, _ = apply_rotary_pos_emb(x[None, None], x[None, None], cos, sin)
    return q[0, 0].numpy()


@pytest.mark.parametrize("d,base", [(64, 1e4), (128, 1e4), (128, 5e5)])
def test_rope_matches_transformers(d, base):
    rng = np.random.default_rng(0)
    x = rng.standard_normal((50, d))
    pos = rng.integers(0, 40000, 50)
    # the two ways of forming base^(-2i/d) differ by a few fp64 ulp; times a
    # position up to 4e4 that moves the angle by ~1e-11 rad
    np.testing.assert_allclose(O.rope(x, pos, base), hf_rope(x, pos, base), atol=1e-10, rtol=0)


def test_rope_shift_invariance():
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal((1, 128)), rng.standard_normal((30, 128))
    pk = np.arange(30)
    s0 = O.rope(k, pk, 1e4) @ O.rope(q, [29], 1e4)[0]
    s1 = O.rope(k, pk + 12345, 1e4) @ O.rope(q, [29 + 12345], 1e4)[0]
    np.testing.assert_allclose(s0, s1, atol=1e-10)


def _rand_case(H=4, h_kv=2, d=64, r_k=16, R=64, n=37, seed=0, m=1):
    rng = np.random.default_rng(seed)
    cfg = O.Config(H=H, h_kv=h_kv, d_h=d, hidden=8, r_k=r_k, R=R)
    zk = rng.standard_normal((n, h_kv, r_k))
    zv = rng.standard_normal((n, R))
    Bk = rng.standard_normal((h_kv, r_k, d)) / np.sqrt(r_k)
    Bv = rng.standard_normal((R, h_kv * d)) / np.sqrt(R)
    q = rng.standard_normal((m, H, d))
    return cfg, zk, zv, Bk, Bv, q


def _sdpa_materialised(cfg, zk, zv, Bk, Bv, q, q_pos):
    """Brute force: decompress the full K (RoPE'd) and V per head, then SDPA."""
    n = zk.shape[0]
    d = cfg.d_h
    K = np.stack([hf_rope(zk[:, kv] @ Bk[kv], np.arange(n), cfg.rope_base) for kv in range(cfg.h_kv)])
    V = np.stack([zv @ Bv[:, kv * d:(kv + 1) * d] for kv in range(cfg.h_kv)])
    Q = np.stack([hf_rope(q[:, h], q_pos, cfg.rope_base) for h in range(cfg.H)])      # [H, m, d]
    mask = torch.as_tensor(np.arange(n)[None, :] <= np.asarray(q_pos)[:, None])
    o = F.scaled_dot_product_attention(torch.as_tensor(Q)[None], torch.as_tensor(K)[None],
                                       torch.as_tensor(V)[None], attn_mask=mask,
                                       enable_gqa=cfg.H != cfg.h_kv)
    return o[0].numpy().transpose(1, 0, 2)                                           # [m, H, d]


@pytest.mark.parametrize("H,h_kv", [(4, 4), (8, 2)])
def test_reassociated_equals_materialised(H, h_kv):
    # [Review] eq. 12: p_h (Z_V U_h^T) = (p_h Z_V) U_h^T, plus GQA head mapping
    cfg, zk, zv, Bk, Bv, q = _rand_case(H=H, h_kv=h_kv, m=5, n=70)
    q_pos = np.array([69, 3, 40, 0, 69])
    got = O.attend_latents(cfg, zk, zv, q, q_pos, Bk, Bv)
    ref = _sdpa_materialised(cfg, zk, zv, Bk, Bv, q, q_pos)
    np.testing.assert_allclose(got, ref, atol=1e-12, rtol=0)


@pytest.mark.parametrize("rotate", [False, True])
def test_full_rank_latents_reproduce_dense_attention(rotate):
    # r_k = d_h, R = h_kv d_h, orthonormal B: latent attention == dense attention
    # with W_k = A_k B_k, W_v = A_v B_v; the block rotation (eq. 13) changes nothing.
    rng = np.random.default_rng(7)
    H, h_kv, d, hidden, n = 4, 2, 32, 48, 25
    cfg = O.Config(H=H, h_kv=h_kv, d_h=d, hidden=hidden, r_k=d, R=h_kv * d)
    X = rng.standard_normal((n, hidden))
    A_k = rng.standard_normal((hidden, h_kv * d)) / np.sqrt(hidden)
    A_v = rng.standard_normal((hidden, h_kv * d)) / np.sqrt(hidden)
    Bk = np.stack([np.linalg.qr(rng.standard_normal((d, d)))[0].T for _ in range(h_kv)])
    Bv = np.linalg.qr(rng.standard_normal((h_kv * d, h_kv * d)))[0].T
    q = rng.standard_normal((1, H, d))
    zk = (X @ A_k).reshape(n, h_kv, d)
    zv = X @ A_v
    if rotate:
        g = cfg.key.g
        zk = O.unrotate_fp64(zk.reshape(n, -1) @ np.kron(np.eye(h_kv * d // g), O.hadamard_fp64(g)), g).reshape(n, h_kv, d)
        zv = O.unrotate_fp64(zv @ np.kron(np.eye(h_kv * d // cfg.val.g), O.hadamard_fp64(cfg.val.g)), cfg.val.g)
    got = O.attend_latents(cfg, zk, zv, q, [n - 1], Bk, Bv)
    Wk = [A_k[:, kv * d:(kv + 1) * d] @ Bk[kv] for kv in range(h_kv)]
    Wv = A_v @ Bv
    K = np.stack([hf_rope(X @ Wk[kv], np.arange(n), cfg.rope_base) for kv in range(h_kv)])
    V = np.stack([X @ Wv[:, kv * d:(kv + 1) * d] for kv in range(h_kv)])
    Q = np.stack([hf_rope(q[:, h], [n - 1], cfg.rope_base) for h in range(H)])
    o = F.scaled_dot_product_attention(torch.as_tensor(Q)[None], torch.as_tensor(K)[None],
                                       torch.as_tensor(V)[None], enable_gqa=True)[0].numpy()
    np.testing.assert_allclose(got, o.transpose(1, 0, 2), atol=1e-12, rtol=0)


def test_partition_identity_merge():
    # [CaliDrop] eq. 1: Att over a partition = alpha-weighted sum of subset attentions
    rng = np.random.default_rng(8)
    s = rng.standard_normal(1000) * 4
    v = rng.standard_normal((1000, 33))
    p = np.exp(s - s.max())
    ref = p @ v / p.sum()
    for cuts in ([], [1], [500], [3, 3, 999], sorted(rng.choice(999, 7, replace=False) + 1)):
        b = [0] + list(cuts) + [1000]
        parts = [O.partial_softmax(s[lo:hi], v[lo:hi]) for lo, hi in zip(b[:-1], b[1:])]
        np.testing.assert_allclose(O.lse_merge(parts), ref, atol=1e-13, rtol=0)


def test_single_token_returns_its_value():
    cfg, zk, zv, Bk, Bv, q = _rand_case(n=1)
    got = O.attend_latents(cfg, zk, zv, q, [0], Bk, Bv)
    for h in range(cfg.H):
        kv = h // cfg.group
        np.testing.assert_allclose(got[0, h], zv[0] @ Bv[:, kv * 64:(kv + 1) * 64], atol=1e-13)


def test_identical_keys_average_values():
    cfg, zk, zv, Bk, Bv, q = _rand_case(n=20)
    # identical *pre-RoPE* keys still differ after RoPE; take d_h-invariant keys: zero keys
    zk[:] = 0.0
    got = O.attend_latents(cfg, zk, zv, q, [19], Bk, Bv)
    for h in range(cfg.H):
        kv = h // cfg.group
        np.testing.assert_allclose(got[0, h], zv.mean(0) @ Bv[:, kv * 64:(kv + 1) * 64], atol=1e-13)


def test_decode_through_paged_cache_equals_direct():
    # gather through a shuffled block table == dequantising the pages in order
    w = gen.shrink(gen.workload(0), ctx=77)
    cfg = O.config_of(w)
    f = gen.make_factors(w)
    zk, zv = gen.make_latents(w, 77)
    bt, n_pages = gen.make_block_table([77], extra_pages=3)
    cache = O.new_cache(cfg, n_pages)
    O.write_latents(cache, gen.slots_for(bt, 0, np.arange(77)), zk, zv)
    q = gen.make_queries(1, w.H, w.d_h)
    got = O.decode(cache, q, f.B_k, f.B_v, bt, [77])
    ck = [O.quantize_latent(zk[:, h], cfg.key) for h in range(cfg.h_kv)]
    zkh = np.stack([O.dequantize_codes(*c, cfg.key) for c in ck], 1)
    zvh = O.dequantize_codes(*O.quantize_latent(zv, cfg.val), cfg.val)
    ref = _sdpa_materialised(cfg, O.unrotate_fp64(zkh, cfg.key.g), O.unrotate_fp64(zvh, cfg.val.g),
                             f.B_k.astype(np.float64), f.B_v.astype(np.float64), q.astype(np.float64), [76])
    np.testing.assert_allclose(got, ref, atol=1e-12, rtol=0)


def test_prefill_is_causal_decode_per_query():
    # each prefill query equals a decode whose sequence ends at that query
    w = gen.shrink(gen.workload(0), ctx=50)
    cfg = O.config_of(w)
    f = gen.make_factors(w)
    zk, zv = gen.make_latents(w, 50)
    bt, n_pages = gen.make_block_table([50])
    cache = O.new_cache(cfg, n_pages)
    O.write_latents(cache, gen.slots_for(bt, 0, np.arange(50)), zk, zv)
    q = gen.make_queries(9, w.H, w.d_h)
    got = O.prefill(cache, q, [0, 9], f.B_k, f.B_v, bt, [50])
    for i in range(9):
        d = O.decode(cache, q[i:i + 1], f.B_k, f.B_v, bt, [42 + i])   # query at 41 + i
        np.testing.assert_allclose(got[i], d[0], atol=1e-13)


def test_quantised_attention_close_to_unquantised():
    # sanity: 4/3-bit latents perturb the output a little, not grossly
    w = gen.shrink(gen.workload(0), ctx=256)
    cfg = O.config_of(w)
    f = gen.make_factors(w)
    zk, zv = gen.make_latents(w, 256)
    bt, n_pages = gen.make_block_table([256])
    cache = O.new_cache(cfg, n_pages)
    O.write_latents(cache, gen.slots_for(bt, 0, np.arange(256)), zk, zv)
    q = gen.make_queries(1, w.H, w.d_h)
    got = O.decode(cache, q, f.B_k, f.B_v, bt, [256])
    ref = O.attend_latents(cfg, zk, zv, q, [255], f.B_k, f.B_v)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 0.2


def test_empty_sequence_decodes_to_zero_row():
    w = gen.workload(0)
    cfg = O.config_of(w)
    f = gen.make_factors(w)
    cache = O.new_cache(cfg, 1)
    q = gen.make_queries(1, w.H, w.d_h)
    assert np.all(O.decode(cache, q, f.B_k, f.B_v, np.zeros((1, 1), np.int32), [0]) == 0)


def _slice_case(w, n, cuts, seed=0):
    """One sequence of n tokens written whole into one cache and, slice by slice,
    into one cache per slice (each slice's pages from local index 0)."""
    cfg = O.config_of(w)
    zk, zv = gen.make_latents(w, n, seed)
    bt, n_pages = gen.make_block_table([n], seed)
    whole = O.new_cache(cfg, n_pages)
    O.write_latents(whole, gen.slots_for(bt, 0, np.arange(n)), zk, zv)
    slices = []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        sbt, sp = gen.make_block_table([max(hi - lo, 1)], seed + lo + 1)
        c = O.new_cache(cfg, sp)
        if hi > lo:
            O.write_latents(c, gen.slots_for(sbt, 0, np.arange(hi - lo)), zk[lo:hi], zv[lo:hi])
        slices.append((c, sbt, lo, hi))
    return cfg, whole, bt, slices


@pytest.mark.parametrize("wi", [0, 3])
def test_slices_merge_to_the_whole_decode(wi):
    # [CaliDrop] eq. 1 (partition identity): the query attends to disjoint key
    # slices at their own positions and the merged result is the whole decode
    w = gen.workload(wi)
    n = 300
    cuts = [0, 100, 100, 251, 300]                  # includes an empty slice
    cfg, whole, bt, slices = _slice_case(w, n, cuts)
    f = gen.make_factors(w)
    q = gen.make_queries(1, w.H, w.d_h, seed=3)
    ref = O.decode(whole, q, f.B_k, f.B_v, bt, [n])
    parts = [O.decode_slice(c, q, f.B_k, f.B_v, sbt, [hi - lo], [lo], [n - 1]) for c, sbt, lo, hi in slices]
    o = O.merge_slices([p[0] for p in parts], [p[1] for p in parts], [p[2] for p in parts])
    np.testing.assert_allclose(o, ref, atol=1e-12, rtol=0)
    # the empty slice has (o, m, l) = (0, -inf, 0)
    assert np.all(parts[1][0] == 0) and np.all(parts[1][1] == -np.inf) and np.all(parts[1][2] == 0)


def test_slice_statistics_against_materialised_scores():
    # (m, l) of a slice from scores formed on fully materialised keys RoPE'd by the
    # transformers helper at the slice's global positions
    w = gen.workload(0)
    n, lo, hi = 200, 60, 170
    cfg, whole, bt, slices = _slice_case(w, n, [0, lo, hi, n])
    f = gen.make_factors(w)
    q = gen.make_queries(1, w.H, w.d_h, seed=5)
    c, sbt, _, _ = slices[1]
    o, m, l = O.decode_slice(c, q, f.B_k, f.B_v, sbt, [hi - lo], [lo], [n - 1])
    zk, zv = O.gather_sequence(c, sbt[0], hi - lo)
    zk = O.unrotate_fp64(zk, cfg.key.g)
    zv = O.unrotate_fp64(zv, cfg.val.g)
    for h in range(w.H):
        kv = h // cfg.group
        K = hf_rope(zk[:, kv] @ np.asarray(f.B_k[kv], np.float64), np.arange(lo, hi), cfg.rope_base)
        qr = hf_rope(np.asarray(q[:, h], np.float64), [n - 1], cfg.rope_base)[0]
        s = K @ qr / np.sqrt(w.d_h)
        assert m[0, h] == pytest.approx(s.max(), abs=1e-12)
        assert l[0, h] == pytest.approx(np.exp(s - s.max()).sum(), rel=1e-12)
        p = np.exp(s - s.max()) / np.exp(s - s.max()).sum()
        V = zv @ np.asarray(f.B_v, np.float64)[:, kv * w.d_h:(kv + 1) * w.d_h]
        np.testing.assert_allclose(o[0, h], p @ V, atol=1e-12, rtol=0)


def test_one_slice_is_the_whole_decode():
    w = gen.workload(1)
    w = gen.shrink(w, ctx=64)
    n = 70
    cfg, whole, bt, slices = _slice_case(w, n, [0, n])
    f = gen.make_factors(w)
    q = gen.make_queries(1, w.H, w.d_h, seed=7)
    c, sbt, _, _ = slices[0]
    o, m, l = O.decode_slice(c, q, f.B_k, f.B_v, sbt, [n], [0], [n - 1])
    np.testing.assert_allclose(o, O.decode(whole, q, f.B_k, f.B_v, bt, [n]), atol=1e-12, rtol=0)


@pytest.mark.parametrize("H,h_kv", [(4, 4), (8, 2)])
def test_output_projection_equals_fused_factor_and_dense(H, h_kv):
    # [Review] eq. 12: p_h (Z_V U_h^T) O_h = (p_h Z_V) (U_h^T O_h).  The oracle's
    # two-stage y = sum_h o_h W_o,h equals the fused factor form (latent row times
    # the offline product B_v,h W_o,h) and the dense form (materialised V, torch
    # SDPA, then W_o)
    cfg, zk, zv, Bk, Bv, q = _rand_case(H=H, h_kv=h_kv, m=1, n=60)
    n, d, model = zk.shape[0], cfg.d_h, 48
    rng = np.random.default_rng(7)
    W_o = rng.standard_normal((H * d, model)) / np.sqrt(H * d)
    bt, n_pages = gen.make_block_table([n])
    cache = O.new_cache(cfg, n_pages)
    # unquantised comparison: write latents and compare against the dequantised ones
    O.write_latents(cache, gen.slots_for(bt, 0, np.arange(n)), zk.astype(np.float32), zv.astype(np.float32))
    y = O.decode_out(cache, q, Bk, Bv, W_o, bt, [n])
    zkh, zvh = O.gather_sequence(cache, bt[0], n)
    zkh, zvh = O.unrotate_fp64(zkh, cfg.key.g), O.unrotate_fp64(zvh, cfg.val.g)
    dense = _sdpa_materialised(cfg, zkh, zvh, Bk, Bv, q, [n - 1]).reshape(1, H * d) @ W_o
    np.testing.assert_allclose(y, dense, atol=1e-12, rtol=0)
    # fused factor: for each head, (p_h Z_v) (B_v[:, kv] W_o,h)
    fused = np.zeros((1, model))
    for h in range(H):
        kv = h // cfg.group
        k = hf_rope(zkh[:, kv] @ Bk[kv], np.arange(n), cfg.rope_base)
        qr = hf_rope(q[:, h], [n - 1], cfg.rope_base)
        s = (qr @ k.T) / np.sqrt(d)
        p = np.exp(s - s.max())
        p /= p.sum()
        F = Bv[:, kv * d:(kv + 1) * d] @ W_o[h * d:(h + 1) * d]
        fused += (p @ zvh) @ F
    np.testing.assert_allclose(y, fused, atol=1e-12, rtol=0)


@pytest.mark.parametrize("wi", [0, 3])
def test_fp16_variant_attention_close_to_unquantised(wi):
    # the unquantised variant differs from exact latents only by fp16 rounding of
    # the rotated values (relative 2^-11): far tighter than the 4/3-bit cache
    w = gen.shrink(gen.workload(wi), ctx=200, fp16_latent=True)
    cfg = O.config_of(w)
    f = gen.make_factors(w)
    zk, zv = gen.make_latents(w, 200)
    bt, n_pages = gen.make_block_table([200])
    cache = O.new_cache(cfg, n_pages)
    O.write_latents(cache, gen.slots_for(bt, 0, np.arange(200)), zk, zv)
    q = gen.make_queries(1, w.H, w.d_h)
    got = O.decode(cache, q, f.B_k, f.B_v, bt, [200])
    ref = O.attend_latents(cfg, zk, zv, q, [199], f.B_k, f.B_v)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 2e-3
    # and the 4/3-bit cache of the same latents is much further off
    w43 = gen.shrink(w, fp16_latent=False)
    c43 = O.new_cache(O.config_of(w43), n_pages)
    O.write_latents(c43, gen.slots_for(bt, 0, np.arange(200)), zk, zv)
    rel43 = np.linalg.norm(O.decode(c43, q, f.B_k, f.B_v, bt, [200]) - ref) / np.linalg.norm(ref)
    assert rel43 > 4 * rel


def test_ragged_ranks_decode_against_materialised():
    # ragged key ranks ([Review] section 3: learned per head): each head's keys
    # are its own r_h latents times its own B_k rows; brute force on the
    # dequantised latents (per-head rotation undone) with torch SDPA
    ranks = (64, 48, 32, 16, 64, 32, 48, 16)
    w = gen.shrink(gen.workload(3), key_ranks=ranks, ctx=90)
    cfg = O.config_of(w)
    f = gen.make_factors(w)
    Bk = O.pad_key_factor(cfg, f.B_k)
    zk, zv = gen.make_latents(w, 90)
    bt, n_pages = gen.make_block_table([90])
    cache = O.new_cache(cfg, n_pages)
    O.write_latents(cache, gen.slots_for(bt, 0, np.arange(90)), zk, zv)
    q = gen.make_queries(1, w.H, w.d_h)
    got = O.decode(cache, q, Bk, f.B_v, bt, [90])
    zkh, zvh = O.gather_sequence(cache, bt[0], 90)
    Kh = np.zeros((90, cfg.h_kv, cfg.r_k))
    for h, r in enumerate(ranks):      # per-head unrotation with the head's own group size
        g = O.latent_split(r).g
        Kh[:, h, :r] = (zkh[:, h, :r].astype(np.float64).reshape(90, r // g, g) @ O.hadamard_fp64(g)).reshape(90, r)
    ref = _sdpa_materialised(cfg, Kh, O.unrotate_fp64(zvh, cfg.val.g), Bk, f.B_v, q, [89])
    np.testing.assert_allclose(got, ref, atol=1e-12, rtol=0)
    # padded channels carry nothing: the padded B_k rows are zero
    for h, r in enumerate(ranks):
        assert np.all(Bk[h, r:] == 0)
