"""Byte accounting pins: the layout's bytes against the review's closed forms.

[Review] eq. 1 (dense payload), eq. 14 (mean bits, payload compression),
eq. 15 (latent payload), eq. 16 (exempt-layer fraction).  The printed values
live in tests/golden/review_numbers.json.
"""
import json
import os

import numpy as np
import pytest

import oracle as O
from harness import gen

NUM = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "review_numbers.json")))


def test_eq14_printed_values():
    assert O.eq14_mean_bits(0.2) == pytest.approx(NUM["eq14_mean_bits_top20"]["value"], abs=1e-12)
    assert O.eq14_payload_compression(0.25, 3.2) == pytest.approx(NUM["eq14_payload_compression_rho0.25"]["value"])
    assert O.eq14_payload_compression(0.4, 3.2) == pytest.approx(NUM["eq14_payload_compression_rho0.4"]["value"])


def test_eq16_printed_values():
    f = O.eq16_retained_fraction()
    assert f == pytest.approx(NUM["eq16_retained_fraction"]["value"], abs=1e-15)
    assert 1 / f == pytest.approx(NUM["eq16_inverse"]["value"], abs=NUM["eq16_inverse"]["tol"])


@pytest.mark.parametrize("i", range(5))
def test_layout_payload_equals_eq15(i):
    w = gen.workload(i)
    cfg = O.config_of(w)
    mean_bits = O.eq14_mean_bits(w.top_fraction)            # 3.25 at top_fraction 0.25
    eq15 = O.eq15_latent_payload_bytes(1, 1, mean_bits, [[w.r_k] * w.h_kv], [w.R])
    assert O.payload_bytes_per_token(cfg) == pytest.approx(eq15, abs=1e-12)
    # metadata: one fp16 (scale, zero) pair per group per token; padding explicit
    meta = 4 * (w.h_kv * w.r_k // cfg.key.g + w.R // cfg.val.g)
    pad = w.h_kv * (cfg.key.region_bytes - cfg.key.payload_bytes) / 16 + (cfg.val.region_bytes - cfg.val.payload_bytes) / 16
    assert O.cache_bytes_per_token(cfg) == pytest.approx(eq15 + meta + pad, abs=1e-12)


def test_longchat_payload_ratio_against_eq1():
    # rank fraction 0.25 of 2 h_kv d_h channels at 3.25 bits vs an fp16 cache: 16/(0.25*3.25)
    w = gen.workload(1)
    cfg = O.config_of(w)
    dense = O.eq1_dense_payload_bytes(1, 1, 1, w.h_kv, w.d_h, 16)
    assert dense / O.payload_bytes_per_token(cfg) == pytest.approx(16 / (0.25 * 3.25), rel=1e-12)
    # the review's 20x at 3.2 bits is reproduced by a 20:80 split
    w2 = gen.shrink(w, top_fraction=0.2)
    r = (w2.h_kv * w2.r_k + w2.R) / (2 * w2.h_kv * w2.d_h)
    assert O.eq14_payload_compression(r, O.eq14_mean_bits(0.2)) == pytest.approx(20.0)


def test_known_per_token_bytes():
    # LongChat-7B shapes: 416 key payload + 512 key meta + 416 value payload + 256 value meta
    assert O.cache_bytes_per_token(O.config_of(gen.workload(1))) == 1600
    assert O.cache_bytes_per_token(O.config_of(gen.workload(3))) == 672


RAGGED = (64, 48, 32, 16, 64, 32, 48, 16)


def _ragged(i=3, ranks=RAGGED):
    return gen.shrink(gen.workload(i), key_ranks=ranks)


def test_ragged_payload_equals_eq15():
    # [Review] eq. 15 with per-head ranks: (B T b/8) (sum_h r^K_h + R^V); each rank is
    # a multiple of 16, so its 4-bit block is exactly a quarter (b = 3.25 per channel)
    w = _ragged()
    cfg = O.config_of(w)
    eq15 = O.eq15_latent_payload_bytes(1, 1, O.eq14_mean_bits(0.25), [list(RAGGED)], [w.R])
    assert O.payload_bytes_per_token(cfg) == pytest.approx(eq15, abs=1e-12)
    # per-page strides: each head's region (payload padded to 16 B) and one
    # (scale, zero) word per group of 16 tokens, with the head's own group size
    region = lambda r: (2 * (4 * (r // 4) + 3 * (r - r // 4)) + 15) // 16 * 16
    gsize = {16: 4, 32: 8, 48: 4, 64: 16}                  # gcd(16, r/4, 3r/4) by hand
    heads, kb, km = cfg.key_layout()
    assert kb == sum(region(r) for r in RAGGED)
    assert km == sum(16 * r // gsize[r] for r in RAGGED)
    assert [cfg.key_head(h).g for h in range(len(RAGGED))] == [gsize[r] for r in RAGGED]
    offs = np.concatenate([[0], np.cumsum([region(r) for r in RAGGED])])[:-1]
    assert [c for _, c, _ in heads] == list(offs)
    sizes = O.layout_sizes(cfg, 3)
    assert sizes["k_codes"] == 3 * kb and sizes["k_meta"] == 3 * km * 4


def test_ragged_pages_hold_each_heads_own_codes():
    # the flat key page of a ragged cache, cut at offsets computed by hand, holds
    # each head's latents quantised with that head's own geometry
    w = _ragged()
    cfg = O.config_of(w)
    n = 40
    zk, zv = gen.make_latents(w, n, seed=4)
    bt, n_pages = gen.make_block_table([n], seed=4)
    cache = O.new_cache(cfg, n_pages)
    O.write_latents(cache, gen.slots_for(bt, 0, np.arange(n)), zk, zv)
    pages = bt[0, :(n + 15) // 16]
    code_off, meta_off = 0, 0
    for h, r in enumerate(RAGGED):
        lat = O.latent_split(r, 0.25)
        c, s, zp = O.quantize_latent(zk[:, h, :r], lat)
        P = len(pages)
        cc = np.zeros((P * 16, r), np.uint8)
        ss = np.zeros((P * 16, lat.n_groups), np.float16)
        zz = np.zeros((P * 16, lat.n_groups), np.float16)
        cc[:n], ss[:n], zz[:n] = c, s, zp
        want_b, want_m = O.pack_region(cc, ss, zz, lat)
        got_b = cache.k_codes[pages, code_off:code_off + lat.region_bytes]
        got_m = cache.k_meta[pages, meta_off:meta_off + lat.n_groups * 16].reshape(P, lat.n_groups, 16)
        np.testing.assert_array_equal(got_b, want_b)
        np.testing.assert_array_equal(got_m, want_m)
        code_off += lat.region_bytes
        meta_off += lat.n_groups * 16


def test_uniform_rank_table_is_the_uniform_layout():
    # a table of equal ranks stores the same bytes as the uniform configuration
    w = gen.workload(1)
    wr = gen.shrink(w, key_ranks=(w.r_k,) * w.h_kv, ctx=64)
    cu, cr = O.config_of(gen.shrink(w, ctx=64)), O.config_of(wr)
    n = 33
    zk, zv = gen.make_latents(gen.shrink(w, ctx=64), n)
    bt, n_pages = gen.make_block_table([n])
    a, b = O.new_cache(cu, n_pages), O.new_cache(cr, n_pages)
    O.write_latents(a, gen.slots_for(bt, 0, np.arange(n)), zk, zv)
    O.write_latents(b, gen.slots_for(bt, 0, np.arange(n)), zk, zv)
    np.testing.assert_array_equal(a.k_codes.reshape(n_pages, -1), b.k_codes)
    np.testing.assert_array_equal(a.k_meta.reshape(n_pages, -1), b.k_meta)
