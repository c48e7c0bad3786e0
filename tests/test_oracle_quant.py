"""Pins of the oracle's rotation, quantiser and packed layout (CPU only).

Each test checks the oracle against something other than itself: scipy's
Hadamard matrix, an error bound, brute-force nearest-grid search, exhaustive
enumeration, or hand-derived byte images stored in tests/golden/.
"""
import json
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import scipy.linalg

import oracle as O
from harness import gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("g", [1, 2, 4, 8, 16])
def test_hadamard_matches_scipy(g):
    # [Review] eq. 13: H is orthogonal block-diagonal; Sylvester construction.
    H = O.hadamard_fp64(g)
    np.testing.assert_array_equal(H * np.sqrt(g), scipy.linalg.hadamard(g))
    np.testing.assert_allclose(H @ H, np.eye(g), atol=1e-15)


def test_inv_sqrt_constant_is_correctly_rounded():
    getcontext().prec = 60
    for g in (1, 2, 4, 8, 16):
        exact = Decimal(1) / Decimal(g).sqrt()
        c = O.inv_sqrt_fl32(g)
        # the nearest binary32: its neighbours must be no closer
        up = np.nextafter(c, np.float32(1))
        dn = np.nextafter(c, np.float32(0))
        err = abs(Decimal(float(c)) - exact)
        assert err <= abs(Decimal(float(up)) - exact)
        assert err <= abs(Decimal(float(dn)) - exact)


@pytest.mark.parametrize("g", [4, 8, 16])
def test_fwht_within_fp32_bound_of_matrix_product(g):
    rng = np.random.default_rng(1)
    z = (rng.standard_normal((200, 4 * g)) * rng.uniform(0.01, 30, size=(200, 1))).astype(np.float32)
    got = O.rotate_fl32(z, g).astype(np.float64)
    ref = (z.astype(np.float64).reshape(200, 4, g) @ scipy.linalg.hadamard(g) / np.sqrt(g)).reshape(200, 4 * g)
    # log2(g) butterfly roundings + 1 scale rounding, each <= 2^-24 relative of a partial sum
    bound = (np.log2(g) + 2) * 2.0 ** -24 * (np.abs(z).reshape(200, 4, g).sum(-1, keepdims=True)
                                            * np.ones((1, 1, g))).reshape(200, 4 * g)
    assert np.all(np.abs(got - ref) <= bound)
    # and the rotation is undone by the fp64 inverse up to the same bound
    back = O.unrotate_fp64(got, g)
    assert np.all(np.abs(back - z) <= 2 * bound)


def _one_group(bits, g=16):
    """Geometry of a latent that is a single group of g channels at `bits` bits."""
    return O.Latent(g, g if bits == 4 else 0, 0 if bits == 4 else g, g)


def test_constant_group_has_zero_scale():
    z = np.full((3, 8), 1.2345678, np.float32)
    codes, s, zp = O.quantize_groups(z, 3)
    assert np.all(s == 0) and np.all(codes == 0)
    zh = O.dequantize_codes(codes, s[:, None], zp[:, None], _one_group(3, 8))
    np.testing.assert_array_equal(zh, np.float16(np.float32(1.2345678)).astype(np.float32))


@pytest.mark.parametrize("bits", [3, 4])
def test_grid_values_round_trip(bits):
    rng = np.random.default_rng(2)
    qmax = 2 ** bits - 1
    for _ in range(200):
        s = np.float16(rng.uniform(1e-3, 2.0))
        zp = np.float16(rng.uniform(-5, 5))
        k = rng.integers(0, qmax + 1, size=16)
        k[0], k[1] = 0, qmax                     # both ends present -> range = qmax * s
        z = (k.astype(np.float32) * np.float32(s) + np.float32(zp)).astype(np.float32)
        codes, s2, zp2 = O.quantize_groups(z[None], bits)
        if np.float32(z.max()) - np.float32(z.min()) != np.float32(qmax) * np.float32(s):
            continue                             # range not exact in fp32 (rare); skip
        assert s2[0] == s and zp2[0] == zp
        np.testing.assert_array_equal(codes[0], k)
        # values on the grid come back exactly through the dequantiser: k s + zp
        back = O.dequantize_codes(codes, s2[:, None], zp2[:, None], _one_group(bits))
        np.testing.assert_array_equal(back[0], z)


@pytest.mark.parametrize("bits", [3, 4])
def test_codes_are_nearest_grid_point_bruteforce(bits):
    rng = np.random.default_rng(3)
    z = (rng.standard_normal((500, 16)) * rng.uniform(0.01, 20, (500, 1))).astype(np.float32)
    codes, s, zp = O.quantize_groups(z, bits)
    qmax = 2 ** bits - 1
    assert codes.max() <= qmax
    grid = np.arange(qmax + 1)[None, None, :] * s.astype(np.float64)[:, None, None] + zp.astype(np.float64)[:, None, None]
    dist = np.abs(z.astype(np.float64)[..., None] - grid)            # [500, 16, qmax+1]
    chosen = np.take_along_axis(dist, codes[..., None].astype(np.int64), -1)[..., 0]
    best = dist.min(-1)
    # the chosen point is the nearest up to the fp32 rounding of (z - zp) / s
    tol = 4 * 2.0 ** -23 * (np.abs(z) + np.abs(zp.astype(np.float64))[:, None] + s.astype(np.float64)[:, None] * qmax)
    assert np.all(chosen - best <= tol)


@pytest.mark.parametrize("bits", [3, 4])
def test_quantisation_error_bound(bits):
    rng = np.random.default_rng(4)
    z = (rng.standard_normal((1000, 16)) * rng.uniform(0.01, 50, (1000, 1))).astype(np.float32)
    codes, s, zp = O.quantize_groups(z, bits)
    zh = codes.astype(np.float32) * s.astype(np.float32)[:, None] + zp.astype(np.float32)[:, None]
    mn, mx = z.min(1).astype(np.float64), z.max(1).astype(np.float64)
    qmax = 2 ** bits - 1
    s64 = s.astype(np.float64)
    s_exact = (mx - mn) / qmax
    bound = (s64 / 2 + np.abs(mn - zp.astype(np.float64)) + qmax * np.abs(s64 - s_exact)
             + 8 * 2.0 ** -24 * (np.abs(mx) + np.abs(mn)))
    err = np.abs(zh.astype(np.float64) - z).max(1)
    assert np.all(err <= bound)


@pytest.mark.parametrize("r,frac", [(16, 0.25), (32, 0.25), (64, 0.25), (512, 0.25), (1024, 0.25)])
def test_pack_unpack_exhaustive(r, frac):
    lat = O.latent_split(r, frac)
    rng = np.random.default_rng(5)
    P = 3
    # every code value at every (token, channel) position across pages
    codes = np.empty((P * 16, r), np.uint8)
    for ch in range(r):
        bits = 4 if ch < lat.n_top else 3
        codes[:, ch] = (np.arange(P * 16) + ch) % (2 ** bits)
    s = rng.standard_normal((P * 16, lat.n_groups)).astype(np.float16)
    zp = rng.standard_normal((P * 16, lat.n_groups)).astype(np.float16)
    data, meta = O.pack_region(codes, s, zp, lat)
    assert data.shape == (P, lat.region_bytes)
    c2, s2, z2 = O.unpack_region(data, meta, lat)
    np.testing.assert_array_equal(c2, codes)
    np.testing.assert_array_equal(s2.view(np.uint16), s.view(np.uint16))
    np.testing.assert_array_equal(z2.view(np.uint16), zp.view(np.uint16))


def test_pack_matches_hand_derived_bytes():
    spec = json.load(open(os.path.join(GOLDEN, "pack_bits.json")))
    for case in spec["cases"]:
        lat = O.latent_split(case["r"], 0.25)
        assert (lat.n_top, lat.g, lat.region_bytes) == (case["n_top"], case["g"], case["region_bytes"])
        codes = np.zeros((16, case["r"]), np.uint8)
        for t, c, v in case["codes"]:
            codes[t, c] = v
        z = np.zeros((16, lat.n_groups), np.float16)
        data, _ = O.pack_region(codes, z, z, lat)
        want = np.zeros(lat.region_bytes, np.uint8)
        for k, v in case["bytes"].items():
            want[int(k)] = v
        np.testing.assert_array_equal(data[0], want)
    m = spec["meta_example"]
    _, meta = O.pack_region(np.zeros((16, 16), np.uint8), np.full((16, 4), m["s"], np.float16),
                            np.full((16, 4), m["zp"], np.float16), O.latent_split(16))
    assert int(meta[0, 0, 0]) == m["word"]


def test_group_size_reading():
    # gcd(16, n_top, n_bot): groups never straddle the 4-bit / 3-bit boundary
    assert O.latent_split(16).g == 4
    assert O.latent_split(32).g == 8
    for r in (64, 512, 1024):
        assert O.latent_split(r).g == 16
    for r in (16, 32, 64, 128, 512, 1024):
        lat = O.latent_split(r)
        assert lat.n_top % lat.g == 0 and lat.n_bot % lat.g == 0


def test_write_latents_partial_pages_keep_other_rows():
    rng = np.random.default_rng(6)
    cfg = O.Config(H=2, h_kv=2, d_h=64, hidden=32, r_k=16, R=64)
    cache = O.new_cache(cfg, 4)
    zk = rng.standard_normal((40, 2, 16)).astype(np.float32)
    zv = rng.standard_normal((40, 64)).astype(np.float32)
    slots = rng.permutation(64)[:40]
    O.write_latents(cache, slots[:25], zk[:25], zv[:25])
    O.write_latents(cache, slots[25:], zk[25:], zv[25:])
    one = O.new_cache(cfg, 4)
    O.write_latents(one, slots, zk, zv)
    np.testing.assert_array_equal(cache.k_codes, one.k_codes)
    np.testing.assert_array_equal(cache.v_meta, one.v_meta)
    # each token's stored codes equal quantising that token alone
    for i in (0, 17, 39):
        c, s, z = O.quantize_latent(zv[i:i + 1], cfg.val)
        page, off = divmod(int(slots[i]), 16)
        cc, ss, zz = O.unpack_region(cache.v_codes[page:page + 1], cache.v_meta[page:page + 1], cfg.val)
        np.testing.assert_array_equal(cc[off], c[0])
        np.testing.assert_array_equal(ss[off].view(np.uint16), s[0].view(np.uint16))


def test_quant_error_raises_on_fp16_overflow():
    with pytest.raises(O.QuantError):
        O.quantize_groups(np.array([[0.0, 1e6, 0.0, 0.0]], np.float32), 4)


def test_projection_is_the_correctly_rounded_product():
    # pre-quantisation latent = fl32 of the exact product X A ([Review] section 2.2, eq. 2;
    # the rounding is a reading of the pages).  Cases whose fp64 sums are exact:
    # integers (exact in fp32 as well), a cancellation that fp32 accumulation loses,
    # and a sum just above a rounding tie that fp32 accumulation rounds down.
    rng = np.random.default_rng(9)
    X = rng.integers(-8, 9, (5, 64)).astype(np.float64)
    A = rng.integers(-8, 9, (64, 7)).astype(np.float64)
    exact = [[sum(int(X[i, k]) * int(A[k, j]) for k in range(64)) for j in range(7)] for i in range(5)]
    got = O.project(X, A)
    assert got.dtype == np.float32
    np.testing.assert_array_equal(got, np.array(exact, np.float32))
    X2 = np.array([[1.0, 2.0 ** -30, -1.0], [1.0, 2.0 ** -24, 2.0 ** -26]])
    got2 = O.project(X2, np.ones((3, 1)))
    assert got2[0, 0] == np.float32(2.0 ** -30)
    assert got2[1, 0] == np.float32(1.0 + 2.0 ** -23)


@pytest.mark.parametrize("r", [16, 32, 64, 512, 1024])
def test_quantize_latent_bit_width_per_group(r):
    # [Review] eq. 14 with the card's calibration recipe (top_fraction 0.25,
    # top_bits 4, bottom_bits 3): the leading 25% of a latent's channels, in
    # singular-value order, are the 4-bit block and the rest the 3-bit block.
    # Every group's largest element lands on the top code of its grid, so the
    # largest code of a group tells its width: 15 for a 4-bit group, 7 for a
    # 3-bit group.  The mean width over the channels is then eq. 14's 3.25.
    rng = np.random.default_rng(r)
    lat = O.latent_split(r, 0.25)
    z = (rng.standard_normal((64, r)) * rng.uniform(0.5, 4.0, (64, 1))).astype(np.float32)
    codes, s, zp = O.quantize_latent(z, lat)
    assert codes.shape == (64, r) and s.shape == (64, r // lat.g)
    top_channels = r // 4                                  # 25% of the channels, counted by hand
    width = np.empty(r)
    for c0 in range(0, r, lat.g):
        top = codes[:, c0:c0 + lat.g].max(axis=1)
        want = 15 if c0 < top_channels else 7
        assert np.all(top == want), (c0, np.unique(top))
        assert codes[:, c0:c0 + lat.g].min(axis=1).max() == 0
        width[c0:c0 + lat.g] = 4 if want == 15 else 3
    assert width.mean() == pytest.approx(O.eq14_mean_bits(0.25))
    assert width.mean() == pytest.approx(0.25 * 4 + 0.75 * 3)


def test_quantize_latent_scale_per_group_on_hand_built_input():
    # One token, r = 64 (g = 16): after the rotation, group gi spans a known range.
    # Feed the inverse rotation of a ramp so the rotated values are the ramp
    # itself (up to fp32 rounding of the butterflies, checked below), then the
    # scale of a group is fl16(range / 15) for the first 16 channels (4-bit) and
    # fl16(range / 7) for the other 48 (3-bit).
    lat = O.latent_split(64, 0.25)
    assert (lat.g, lat.n_top) == (16, 16)
    ramp = np.concatenate([np.arange(16, dtype=np.float64) * (gi + 1) * 0.25 - gi for gi in range(4)])
    z = O.unrotate_fp64(ramp[None], 16).astype(np.float32)      # H_g is its own inverse
    zr = O.rotate_fl32(z, 16).astype(np.float64)[0]
    _, s, zp = O.quantize_latent(z, lat)
    for gi in range(4):
        seg = zr[16 * gi:16 * gi + 16]
        qmax = 15 if gi == 0 else 7
        want = np.float16(np.float32(np.float32(seg.max()) - np.float32(seg.min())) / np.float32(qmax))
        assert s[0, gi] == want, gi
        assert zp[0, gi] == np.float16(np.float32(seg.min()))
        # the range is the ramp's (gi + 1) * 0.25 * 15 to within the rotation's rounding
        assert abs((seg.max() - seg.min()) - (gi + 1) * 0.25 * 15) < 1e-4


@pytest.mark.parametrize("r", [16, 64, 512])
def test_uniform_4bit_variant_quantises_every_group_at_4_bits(r):
    # the review's four-bit cache (section 6.1, the speed ablation of section 8.1):
    # top_fraction 1.0 puts every channel in the 4-bit block; mean width 4 bits
    rng = np.random.default_rng(r + 1)
    lat = O.latent_split(r, 1.0)
    assert (lat.n_top, lat.n_bot, lat.g) == (r, 0, 16)
    z = (rng.standard_normal((32, r)) * rng.uniform(0.5, 4.0, (32, 1))).astype(np.float32)
    codes, s, zp = O.quantize_latent(z, lat)
    assert np.all(codes.reshape(32, -1, 16).max(axis=2) == 15)
    assert O.eq14_mean_bits(1.0) == 4.0
    assert lat.payload_bytes == 16 * r * 4 // 8


def test_fp16_variant_page_bytes_by_hand():
    # the unquantised variant's page layout (the library's own specification):
    # group tiles of 16 tokens x 16 channels in channel order, element (t, c) at
    # fp16 index t * 16 + c, little-endian; no metadata
    lat = O.latent_fp16(32)
    assert (lat.g, lat.n_groups, lat.region_bytes, lat.meta_bytes) == (16, 2, 1024, 0)
    v = np.zeros((16, 32), np.float16)
    v[3, 5] = 1.0          # 0x3C00 -> tile 0, index 53 -> bytes 106, 107
    v[0, 18] = -2.0        # 0xC000 -> tile 1, index 2 -> bytes 512 + 4, 5
    v[15, 31] = 0.5        # 0x3800 -> tile 1, index 255 -> bytes 1022, 1023
    data, meta = O.pack_region(v, None, None, lat)
    want = np.zeros(1024, np.uint8)
    want[107], want[517], want[1023] = 0x3C, 0xC0, 0x38
    np.testing.assert_array_equal(data[0], want)
    assert meta.size == 0
    back, _, _ = O.unpack_region(data, None, lat)
    np.testing.assert_array_equal(back.view(np.uint16), v.view(np.uint16))


def test_fp16_variant_keeps_exact_rotated_values():
    # latents whose rotated values are small integers: the rotation is exact in
    # fp32 and every rotated value is an fp16 number, so the store is lossless
    rng = np.random.default_rng(8)
    lat = O.latent_fp16(64)
    k = rng.integers(-300, 301, (20, 64)).astype(np.float64)
    z = O.unrotate_fp64(k, 16).astype(np.float32)          # H_g is its own inverse
    data, _ = O.quantize_pack_region(z, lat)
    zh = O.dequantize_region(data, None, lat, 20)
    np.testing.assert_array_equal(zh, k.astype(np.float32))


def test_fp16_variant_payload_against_eq1():
    # unquantised latents at rank fraction rho: 16-bit payload, compression 1 / rho against eq. 1
    w = gen.workload(1)
    cfg = O.config_of(gen.shrink(w, fp16_latent=True))
    dense = O.eq1_dense_payload_bytes(1, 1, 1, w.h_kv, w.d_h, 16)
    rho = (w.h_kv * w.r_k + w.R) / (2 * w.h_kv * w.d_h)
    assert dense / O.payload_bytes_per_token(cfg) == pytest.approx(1 / rho)
    assert O.cache_bytes_per_token(cfg) == O.payload_bytes_per_token(cfg) == 2 * (w.h_kv * w.r_k + w.R)
