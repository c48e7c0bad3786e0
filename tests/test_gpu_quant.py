"""GPU parity of the rotate/quantise/pack path (bit-exact) and of append."""
import numpy as np
import pytest
import torch

import oracle as O
from harness import gen

from _cases import download, make_ctx, oracle_cache, skv, upload, bf16_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=[0, 1, 3], ids=["tiny", "longchat", "llama3gqa"])
def ctx(request):
    w = gen.shrink(gen.workload(request.param), ctx=64)
    kv, f = make_ctx(w)
    yield w, kv, f
    kv.close()


@pytest.mark.parametrize("which", [0, 1], ids=["key", "value"])
@pytest.mark.parametrize("n", [1, 16, 37, 300])
def test_quantize_pack_bit_exact(ctx, which, n):
    w, kv, _ = ctx
    S = skv()
    cfg = O.config_of(w)
    lat = cfg.key if which == 0 else cfg.val
    rng = np.random.default_rng(n + 10 * which)
    z = (rng.standard_normal((n, lat.r)) * rng.uniform(0.01, 40, (n, 1))
         * np.where(rng.random(lat.r) < 0.05, 8.0, 1.0)).astype(np.float32)
    pages = (n + 15) // 16
    codes = torch.full((pages * lat.region_bytes,), 0xAB, dtype=torch.uint8, device="cuda")
    meta = torch.full((pages * lat.n_groups * 16,), -1, dtype=torch.int32, device="cuda")
    S.starkv_quantize_pack(kv.ctx, which, torch.from_numpy(z).cuda(), codes, meta)
    want_c, want_m = O.quantize_pack_region(z, lat)
    np.testing.assert_array_equal(codes.cpu().numpy().reshape(pages, -1), want_c)
    np.testing.assert_array_equal(meta.cpu().numpy().view(np.uint32).reshape(want_m.shape), want_m)
    # dequantise the oracle's pages on the GPU: bit-exact z_hat
    zh = torch.empty((n, lat.r), dtype=torch.float32, device="cuda")
    S.starkv_dequantize(kv.ctx, which, torch.from_numpy(want_c.reshape(-1)).cuda(),
                        torch.from_numpy(want_m.view(np.int32).reshape(-1)).cuda(), n, zh)
    ref = O.dequantize_region(want_c, want_m, lat, n)
    np.testing.assert_array_equal(zh.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert kv.status() == 0


def test_quantize_edge_groups(ctx):
    # constant groups (scale 0), exact grid values, huge and tiny magnitudes
    w, kv, _ = ctx
    S = skv()
    lat = O.config_of(w).val
    g = lat.g
    z = np.zeros((32, lat.r), np.float32)
    z[0] = 3.25
    z[1] = np.tile(np.arange(g, dtype=np.float32) * 0.125 - 1.0, lat.r // g)
    z[2] = 1e-6 * np.arange(lat.r)
    z[3] = 3e4 * np.sin(np.arange(lat.r))
    z[4, ::7] = -5.0
    codes = torch.zeros(2 * lat.region_bytes, dtype=torch.uint8, device="cuda")
    meta = torch.zeros(2 * lat.n_groups * 16, dtype=torch.int32, device="cuda")
    S.starkv_quantize_pack(kv.ctx, 1, torch.from_numpy(z).cuda(), codes, meta)
    want_c, want_m = O.quantize_pack_region(z, lat)
    np.testing.assert_array_equal(codes.cpu().numpy().reshape(2, -1), want_c)
    np.testing.assert_array_equal(meta.cpu().numpy().view(np.uint32).reshape(want_m.shape), want_m)
    assert kv.status() == 0


def test_quantize_overflow_sets_status(ctx):
    w, kv, _ = ctx
    S = skv()
    lat = O.config_of(w).key
    z = np.zeros((16, lat.r), np.float32)
    z[3, 0] = 1e6       # range / 15 overflows fp16
    codes = torch.zeros(lat.region_bytes, dtype=torch.uint8, device="cuda")
    meta = torch.zeros(lat.n_groups * 16, dtype=torch.int32, device="cuda")
    S.starkv_quantize_pack(kv.ctx, 0, torch.from_numpy(z).cuda(), codes, meta)
    assert kv.status() & S.DEV_QUANT_OVERFLOW
    assert kv.status() == 0    # reading clears it


@pytest.mark.parametrize("n", [1, 7, 16, 45, 300])
def test_append_quantiser_bit_exact_on_exported_latents(ctx, n):
    """The append kernel's quantiser, fed its own fp32 latents, matches the oracle bit for bit."""
    w, kv, f = ctx
    S = skv()
    cfg = O.config_of(w)
    bt, n_pages = gen.make_block_table([n + 5], seed=3, extra_pages=2)
    slots = gen.slots_for(bt, 0, np.arange(5, 5 + n))
    X = gen.make_hidden(n, w.hidden, seed=1)
    lc = kv.new_cache(n_pages)
    lat = torch.zeros((n, w.h_kv * w.r_k + w.R), dtype=torch.float32, device="cuda")
    S.starkv_append(kv.ctx, lc.struct, bf16_tensor(X), torch.from_numpy(slots).cuda(), lat)
    assert kv.status() == 0
    zl = lat.cpu().numpy()
    oc = O.new_cache(cfg, n_pages)
    O.write_latents(oc, slots, zl[:, :w.h_kv * w.r_k].reshape(n, w.h_kv, w.r_k), zl[:, w.h_kv * w.r_k:])
    got = download(lc, oc)
    for name in ("k_codes", "v_codes", "k_meta", "v_meta"):
        np.testing.assert_array_equal(getattr(got, name), getattr(oc, name), err_msg=name)
    # the projection itself: fp32 accumulation of exact bf16 products vs the fp64 product
    ref = np.concatenate([O.project(X, f.A_k), O.project(X, f.A_v)], axis=1)
    bound = 1e-5 * (np.abs(X).astype(np.float64) @ np.abs(np.concatenate([f.A_k, f.A_v], 1))) + 1e-30
    assert np.all(np.abs(zl - ref) <= bound)


PROJ_REL = 1e-5   # projection bound: |z_gpu - z| <= PROJ_REL * (|X| |A|) element-wise (fp32 accumulation)


def _fp16_ulp(v):
    """Spacing of fp16 values at |v| (the subnormal spacing at zero)."""
    e = np.floor(np.log2(np.maximum(np.abs(v.astype(np.float64)), 2.0 ** -14)))
    return 2.0 ** (e - 10)


def test_append_codes_match_oracle_append_bounds():
    # the helper below must reject what it should: a one-ulp shift passes, a
    # shift past the projection bound fails
    s = np.array([[np.float16(0.25)]])
    assert _meta_within(s, s, np.zeros((1, 1)), 15)
    assert _meta_within(np.nextafter(s, np.float16(1)), s, np.zeros((1, 1)), 15)
    assert not _meta_within(s + np.float16(0.01), s, np.full((1, 1), 1e-4), 15)


def _meta_within(got, want, eps, qmax_or_one):
    """|got - want| <= one fp16 ulp plus the shift the projection bound eps can cause."""
    g, w = got.astype(np.float64), want.astype(np.float64)
    return bool(np.all(np.abs(g - w) <= _fp16_ulp(np.maximum(np.abs(g), np.abs(w))) + eps / qmax_or_one + 1e-12))


@pytest.mark.parametrize("n", [64, 200])
def test_append_codes_match_oracle_append(ctx, n):
    """End to end: same X and A on both sides.  The projection's rounding is not
    fixed by the pages (fp32 accumulation on the GPU, the exact product rounded
    once in the oracle), so each latent may differ from the oracle's by the
    projection bound eps = 1e-5 (|X| |A|), which a group's rotation spreads to
    at most sqrt(g) eps.  Each stored scale and zero must then lie within one
    fp16 ulp of the oracle's plus what that shift can cause (2 eps / (2^b - 1)
    for the scale, eps for the zero), and each code must be the one the
    oracle's rotated latent gives under the stored metadata, or differ from it
    by one only where that value's unrounded quotient lies within
    1e-3 + eps / s of a rounding boundary."""
    w, kv, f = ctx
    S = skv()
    cfg = O.config_of(w)
    bt, n_pages = gen.make_block_table([n], seed=4)
    slots = gen.slots_for(bt, 0, np.arange(n))
    X = gen.make_hidden(n, w.hidden, seed=2)
    lc = kv.new_cache(n_pages)
    S.starkv_append(kv.ctx, lc.struct, bf16_tensor(X), torch.from_numpy(slots).cuda())
    oc = O.new_cache(cfg, n_pages)
    zk, zv = O.append(oc, X, f.A_k, f.A_v, slots)
    got = download(lc, oc)
    absXA = np.abs(X).astype(np.float64) @ np.abs(np.concatenate([f.A_k, f.A_v], 1)).astype(np.float64)
    pages, rows = np.unique(slots // 16, return_inverse=True)
    rows = rows * 16 + slots % 16
    kc = w.h_kv * w.r_k
    for h in list(range(w.h_kv)) + [None]:
        lat = cfg.key if h is not None else cfg.val
        z = zk[:, h] if h is not None else zv
        bound = absXA[:, h * w.r_k:(h + 1) * w.r_k] if h is not None else absXA[:, kc:]
        eps = PROJ_REL * np.sqrt(lat.g) * bound.reshape(n, lat.n_groups, lat.g).max(axis=2)   # [n, groups]
        if h is not None:
            parts = [(a[pages, h]) for a in (got.k_codes, got.k_meta, oc.k_codes, oc.k_meta)]
        else:
            parts = [a[pages] for a in (got.v_codes, got.v_meta, oc.v_codes, oc.v_meta)]
        cg, sg, zg = O.unpack_region(parts[0], parts[1], lat)
        co, so, zo = O.unpack_region(parts[2], parts[3], lat)
        cg, sg, zg, so, zo = cg[rows], sg[rows], zg[rows], so[rows], zo[rows]
        zr = O.rotate_fl32(z, lat.g).reshape(n, lat.n_groups, lat.g)
        cgg = cg.reshape(n, lat.n_groups, lat.g).astype(np.int64)
        for lo, hi, bits in ((0, lat.n_top_groups, 4), (lat.n_top_groups, lat.n_groups, 3)):
            if lo == hi:
                continue
            qmax = 2 ** bits - 1
            e = eps[:, lo:hi]
            assert _meta_within(sg[:, lo:hi], so[:, lo:hi], 2 * e, qmax), f"scale, head {h}, {bits}-bit groups"
            assert _meta_within(zg[:, lo:hi], zo[:, lo:hi], e, 1), f"zero, head {h}, {bits}-bit groups"
            want, u = _expected_codes(zr[:, lo:hi], sg[:, lo:hi], zg[:, lo:hi], bits)
            diff = cgg[:, lo:hi] - want
            off = diff != 0
            s64 = sg[:, lo:hi].astype(np.float64)[..., None]
            slack = 1e-3 + np.where(s64 > 0, e[..., None] / np.where(s64 > 0, s64, 1.0), 0.0)
            near = np.abs(u - np.floor(u) - 0.5) < slack
            assert np.all(np.abs(diff) <= 1)
            assert np.all(near[off]), f"code differs away from a rounding boundary ({int(off.sum())} codes)"
    assert kv.status() == 0


def _expected_codes(zr, s, zp, bits):
    """Codes the quantiser gives rotated values zr [n, G, g] under the metadata
    (s, zp) [n, G], and the unrounded fp32 quotients they round from."""
    qmax = np.float32(2 ** bits - 1)
    sf = s.astype(np.float32)[..., None]
    zf = zp.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        u = (zr - zf) / sf
    code = np.where(sf == 0, np.float32(0), np.clip(np.rint(u), np.float32(0), qmax))
    return code.astype(np.int64), np.where(sf == 0, np.float32(0), u)


def test_append_bad_and_negative_slots(ctx):
    w, kv, _ = ctx
    S = skv()
    lc = kv.new_cache(2)
    X = bf16_tensor(gen.make_hidden(3, w.hidden, seed=5))
    slots = torch.tensor([-1, 5, 2 * 16 + 3], dtype=torch.int64, device="cuda")
    S.starkv_append(kv.ctx, lc.struct, X, slots)
    st = kv.status()
    assert st & S.DEV_BAD_SLOT
    # slot 5 was written, the others were not
    assert int(lc.k_meta.view(torch.int32).ne(0).sum()) > 0


def test_general_append_kernel_matches_oracle_quantiser(monkeypatch):
    """The CUDA-core append (taken for large chunks when the tensor-core one is
    switched off): the codes of its exported latents are the oracle's, bit for bit."""
    monkeypatch.setenv("STARKV_APPEND_PATH", "simt")
    w = gen.shrink(gen.workload(1), ctx=64)
    kv, f = make_ctx(w)
    try:
        S = skv()
        cfg = O.config_of(w)
        n = 150
        bt, n_pages = gen.make_block_table([n], seed=5)
        slots = gen.slots_for(bt, 0, np.arange(n))
        X = gen.make_hidden(n, w.hidden, seed=6)
        lc = kv.new_cache(n_pages)
        lat = torch.zeros((n, w.h_kv * w.r_k + w.R), dtype=torch.float32, device="cuda")
        S.starkv_append(kv.ctx, lc.struct, bf16_tensor(X), torch.from_numpy(slots).cuda(), lat)
        assert kv.status() == 0
        zl = lat.cpu().numpy()
        oc = O.new_cache(cfg, n_pages)
        O.write_latents(oc, slots, zl[:, :w.h_kv * w.r_k].reshape(n, w.h_kv, w.r_k), zl[:, w.h_kv * w.r_k:])
        got = download(lc, oc)
        for name in ("k_codes", "v_codes", "k_meta", "v_meta"):
            np.testing.assert_array_equal(getattr(got, name), getattr(oc, name), err_msg=name)
    finally:
        kv.close()
