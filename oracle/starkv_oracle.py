"""fp64 CPU oracle for STAR-KV latent-cache attention (test infrastructure only).

Plain, slow, obviously-correct definitions.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may use this
module; the CUDA library never does.

Notation: fl32 / fl16 = IEEE round-to-nearest-even to binary32 / binary16.
numpy float32 arithmetic rounds every +, -, *, / once, so a float32 numpy
expression *is* the fl32 of each step.

Readings taken where the pages are silent:

* channel split: the first ``round(top_fraction * r)`` channels of a latent
  (singular-value order) are the 4-bit outlier block, the rest the 3-bit
  inlier block ([Review] section 6.1, eq. 14; [Card] calibration recipe,
  top_fraction=0.25, top_bits=4, bottom_bits=3);
* rotation / quantisation group: g = gcd(16, n_top, n_bot) channels, so a
  group never straddles the two blocks, which the review says are rotated
  separately ([Review] section 6.1, eq. 13);
* rotation: normalised Sylvester Hadamard per group, applied as fp32
  butterflies with half-widths 1, 2, 4, ... then one multiply by fl32(1/sqrt g);
* quantiser: asymmetric min/max per (token, group), fp16 scale and fp16 zero
  (= the group minimum), round-half-even, clamp;
* packed layout (see ``pack_region``);
* RoPE: rotate-half pairs (i, i + d/2), theta_i = base^(-2i/d), no position
  scaling ([Review] section 5.3 keeps keys pre-RoPE and rotates at run time);
* output: per-head attention output o_h before the output projection W_o.
"""
from __future__ import annotations

import dataclasses
from math import gcd

import numpy as np

PAGE = 16  # tokens per cache page (16-token KV blocks, as in the paged cache the card's vLLM plugin uses)


class QuantError(ValueError):
    """A group's fp16 scale or zero-point is not finite."""


# ----------------------------------------------------------------------------
# Channel split and group geometry  ([Review] section 6.1, eq. 13-14)
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Latent:
    """Geometry of one latent: a KV head's key latent, or the joint value latent.
    fp16: the unquantised variant ([Review] section 8.1): rotated values stored as fp16."""
    r: int
    n_top: int
    n_bot: int
    g: int
    fp16: bool = False

    @property
    def n_groups(self) -> int:
        return self.r // self.g

    @property
    def n_top_groups(self) -> int:
        return self.n_top // self.g

    def group_bits(self, gi: int) -> int:
        if self.fp16:
            return 16
        return 4 if gi < self.n_top_groups else 3

    @property
    def payload_bytes(self) -> int:
        """Packed bytes of one page (16 tokens): 16 * (4 n_top + 3 n_bot) / 8, or 16 r fp16 values."""
        if self.fp16:
            return 32 * self.r
        return 2 * (4 * self.n_top + 3 * self.n_bot)

    @property
    def region_bytes(self) -> int:
        """Payload padded to a multiple of 16 bytes."""
        return (self.payload_bytes + 15) // 16 * 16

    @property
    def meta_bytes(self) -> int:
        """fp16 (scale, zero) per group per token, for one page (none for fp16 latents)."""
        return 0 if self.fp16 else self.n_groups * PAGE * 4


def latent_split(r: int, top_fraction: float = 0.25) -> Latent:
    """Outlier (4-bit) / inlier (3-bit) split of an r-channel latent ([Review] eq. 14)."""
    n_top = int(np.floor(top_fraction * r + 0.5))
    n_bot = r - n_top
    g = gcd(16, gcd(n_top, n_bot))
    return Latent(r, n_top, n_bot, g)


def latent_fp16(r: int) -> Latent:
    """The unquantised variant ([Review] section 8.1, the unquantised rows of the
    attention-speed ablation): every rotated value stored as fp16; the rotation
    groups are 16 channels (the rotation is exact in real arithmetic and folded
    into the up-projections either way, eq. 13)."""
    return Latent(r, 0, r, 16, True)


@dataclasses.dataclass(frozen=True)
class Config:
    H: int
    h_kv: int
    d_h: int
    hidden: int
    r_k: int
    R: int
    top_fraction: float = 0.25
    rope_base: float = 10000.0
    fp16_latent: bool = False
    key_ranks: tuple = None   # ragged ranks: r_k,h per KV head ([Review] section 3), r_k their maximum

    @property
    def key(self) -> Latent:
        return latent_fp16(self.r_k) if self.fp16_latent else latent_split(self.r_k, self.top_fraction)

    @property
    def ragged(self) -> bool:
        return self.key_ranks is not None

    def key_rank(self, h: int) -> int:
        return self.r_k if self.key_ranks is None else int(self.key_ranks[h])

    def key_head(self, h: int) -> Latent:
        """Geometry of KV head h's key latent (its own rank with ragged ranks)."""
        r = self.key_rank(h)
        return latent_fp16(r) if self.fp16_latent else latent_split(r, self.top_fraction)

    def key_layout(self):
        """Per head (latent column, byte offset in a key-code page, word offset in a
        key-meta page), and the page strides (code bytes, meta words): the heads'
        regions back to back in head order."""
        heads, col, code, meta = [], 0, 0, 0
        for h in range(self.h_kv):
            L = self.key_head(h)
            heads.append((col, code, meta))
            col, code, meta = col + L.r, code + L.region_bytes, meta + L.meta_bytes // 4
        return heads, code, meta

    @property
    def val(self) -> Latent:
        return latent_fp16(self.R) if self.fp16_latent else latent_split(self.R, self.top_fraction)

    @property
    def group(self) -> int:
        return self.H // self.h_kv


def config_of(w) -> Config:
    """Oracle config from a workload description (shape numbers only)."""
    kr = getattr(w, "key_ranks", None)
    return Config(H=w.H, h_kv=w.h_kv, d_h=w.d_h, hidden=w.hidden, r_k=w.r_k, R=w.R,
                  top_fraction=w.top_fraction, rope_base=w.rope_base,
                  fp16_latent=bool(getattr(w, "fp16_latent", False)),
                  key_ranks=tuple(int(r) for r in kr) if kr is not None else None)


# ----------------------------------------------------------------------------
# Projection  ([Review] section 2.2, eq. 2: Z = X V_r Sigma_r, here Z = X A)
# ----------------------------------------------------------------------------
def project(X, A) -> np.ndarray:
    """Pre-quantisation latent: fl32 of the exact (fp64) product X A."""
    return (np.asarray(X, np.float64) @ np.asarray(A, np.float64)).astype(np.float32)


# ----------------------------------------------------------------------------
# Block Hadamard rotation  ([Review] section 6.1, eq. 13; decode dataflow step 2)
# ----------------------------------------------------------------------------
def inv_sqrt_fl32(g: int) -> np.float32:
    """fl32(1/sqrt(g)).  sqrt(g)/g has one fp64 rounding (g a power of two)."""
    return np.float32(np.sqrt(np.float64(g)) / g)


def rotate_fl32(z, g: int) -> np.ndarray:
    """z~ = z H_g for every group of g channels (last axis), in fp32.

    H_g is the Sylvester Hadamard matrix scaled by 1/sqrt(g).  The unscaled
    product is taken by butterflies (a, b) -> (a + b, a - b) over half-widths
    1, 2, 4, ..., each an fp32 add/sub, then one fp32 multiply by fl32(1/sqrt g).
    """
    z = np.asarray(z, np.float32)
    shp = z.shape
    x = z.reshape(-1, shp[-1] // g, g)
    h = 1
    while h < g:
        y = x.reshape(x.shape[0], x.shape[1], g // (2 * h), 2, h)
        a, b = y[..., 0, :], y[..., 1, :]
        x = np.stack([a + b, a - b], axis=-2).reshape(x.shape[0], x.shape[1], g)
        h *= 2
    return (x * inv_sqrt_fl32(g)).reshape(shp)


def hadamard_fp64(g: int) -> np.ndarray:
    """Normalised Sylvester Hadamard matrix H_g (symmetric, H_g H_g = I)."""
    h = np.ones((1, 1))
    while h.shape[0] < g:
        h = np.block([[h, h], [h, -h]])
    return h / np.sqrt(g)


def unrotate_fp64(zr, g: int) -> np.ndarray:
    """Undo the rotation in fp64: z = z~ H_g (H_g is its own inverse), per group."""
    zr = np.asarray(zr, np.float64)
    shp = zr.shape
    x = zr.reshape(-1, shp[-1] // g, g) @ hadamard_fp64(g)
    return x.reshape(shp)


# ----------------------------------------------------------------------------
# Mixed-precision quantiser  ([Review] section 6.1, eq. 14; dataflow step 3)
# ----------------------------------------------------------------------------
def quantize_groups(zr, bits: int):
    """Asymmetric min/max quantiser of fp32 groups (last axis).

    s = fl16(fl32(fl32(mx - mn) / (2^b - 1))), zp = fl16(mn),
    code = clamp(rint_even(fl32(fl32(z - zp) / s)), 0, 2^b - 1), all codes 0 when s == 0.
    Returns (codes uint8 [..., g], s float16 [...], zp float16 [...]).
    """
    zr = np.asarray(zr, np.float32)
    mn = zr.min(axis=-1)
    mx = zr.max(axis=-1)
    qmax = np.float32(2 ** bits - 1)
    with np.errstate(over="ignore"):
        s = ((mx - mn) / qmax).astype(np.float16)
        zp = mn.astype(np.float16)
    if not (np.isfinite(s).all() and np.isfinite(zp).all()):
        raise QuantError("fp16 scale or zero-point overflow")
    sf = s.astype(np.float32)[..., None]
    zf = zp.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        qv = (zr - zf) / sf
    code = np.where(sf == 0, np.float32(0), np.clip(np.rint(qv), np.float32(0), qmax))
    return code.astype(np.uint8), s, zp


def quantize_latent(z, lat: Latent):
    """Rotate then quantise pre-quantisation latents z [n, r] (fp32).

    Returns (codes uint8 [n, r], s float16 [n, G], zp float16 [n, G]) with
    G = r / g groups, codes in the rotated domain.
    """
    z = np.asarray(z, np.float32)
    n = z.shape[0]
    if lat.fp16:
        # unquantised variant: fl16 of the rotated values; no scale or zero
        with np.errstate(over="ignore"):
            v = rotate_fl32(z, lat.g).astype(np.float16)
        if not np.isfinite(v).all():
            raise QuantError("fp16 latent overflow")
        return v, None, None
    zr = rotate_fl32(z, lat.g).reshape(n, lat.n_groups, lat.g)
    codes = np.empty((n, lat.n_groups, lat.g), np.uint8)
    s = np.empty((n, lat.n_groups), np.float16)
    zp = np.empty((n, lat.n_groups), np.float16)
    t = lat.n_top_groups
    if t:
        codes[:, :t], s[:, :t], zp[:, :t] = quantize_groups(zr[:, :t], 4)
    if t < lat.n_groups:
        codes[:, t:], s[:, t:], zp[:, t:] = quantize_groups(zr[:, t:], 3)
    return codes.reshape(n, lat.r), s, zp


def dequantize_codes(codes, s, zp, lat: Latent) -> np.ndarray:
    """z^ = fl32(code * s + zp) per element (rotated domain).  code*s is exact in fp32.
    fp16 latents: the stored fp16 value."""
    if lat.fp16:
        return np.asarray(codes, np.float16).astype(np.float32)
    n = codes.shape[0]
    c = codes.reshape(n, lat.n_groups, lat.g).astype(np.float32)
    zh = c * s.astype(np.float32)[..., None] + zp.astype(np.float32)[..., None]
    return zh.reshape(n, lat.r)


# ----------------------------------------------------------------------------
# Packed page layout (the builder's specification; the pages give none)
# ----------------------------------------------------------------------------
def pack_region(codes, s, zp, lat: Latent):
    """Pack whole pages of one latent region.

    codes [16 P, r] uint8 (rows in page order), s/zp [16 P, G] float16.
    Returns (bytes uint8 [P, region_bytes], meta uint32 [P, G, 16]).

    Layout of one page of one region: group tiles in channel order.  A 4-bit
    tile holds element (t, c) of its 16 x g block at nibble index i = t g + c
    (byte i // 2, low nibble when i is even).  A 3-bit tile is a 2-bit plane of
    the low bits (element i at bits 2 (i mod 4) of byte i // 4) followed by a
    1-bit plane of the high bit (element i at bit i mod 8 of byte i // 8).
    meta[p, group, t] = fp16 scale in the low half, fp16 zero in the high half.
    """
    if lat.fp16:
        # tiles of 16 tokens x g channels in channel order; element (t, c) at fp16 index t g + c
        v = np.asarray(codes, np.float16)
        P = v.shape[0] // PAGE
        tiles = v.reshape(P, PAGE, lat.n_groups, lat.g).transpose(0, 2, 1, 3)       # [P, G, 16, g]
        out = np.ascontiguousarray(tiles).view(np.uint8).reshape(P, lat.region_bytes)
        return out.copy(), np.zeros((P, 0, PAGE), np.uint32)
    codes = np.asarray(codes, np.uint8)
    P = codes.shape[0] // PAGE
    g = lat.g
    c = codes.reshape(P, PAGE, lat.n_groups, g).transpose(0, 2, 1, 3).reshape(P, lat.n_groups, PAGE * g)
    out = np.zeros((P, lat.region_bytes), np.uint8)
    off = 0
    for gi in range(lat.n_groups):
        tile = c[:, gi]
        if lat.group_bits(gi) == 4:
            out[:, off:off + 8 * g] = (tile[:, 0::2] & 0xF) | ((tile[:, 1::2] & 0xF) << 4)
            off += 8 * g
        else:
            lo = tile & 3
            out[:, off:off + 4 * g] = lo[:, 0::4] | (lo[:, 1::4] << 2) | (lo[:, 2::4] << 4) | (lo[:, 3::4] << 6)
            off += 4 * g
            out[:, off:off + 2 * g] = np.packbits((tile >> 2) & 1, axis=1, bitorder="little")
            off += 2 * g
    assert off == lat.payload_bytes
    meta = (np.asarray(s, np.float16).view(np.uint16).astype(np.uint32)
            | (np.asarray(zp, np.float16).view(np.uint16).astype(np.uint32) << 16))
    meta = meta.reshape(P, PAGE, lat.n_groups).transpose(0, 2, 1).copy()
    return out, meta


def unpack_region(data, meta, lat: Latent):
    """Inverse of ``pack_region``: (codes [16 P, r], s [16 P, G], zp [16 P, G])."""
    data = np.asarray(data, np.uint8)
    P = data.shape[0]
    g = lat.g
    if lat.fp16:
        tiles = np.ascontiguousarray(data[:, :lat.payload_bytes]).view(np.float16).reshape(P, lat.n_groups, PAGE, g)
        return tiles.transpose(0, 2, 1, 3).reshape(P * PAGE, lat.r).copy(), None, None
    c = np.empty((P, lat.n_groups, PAGE * g), np.uint8)
    off = 0
    for gi in range(lat.n_groups):
        if lat.group_bits(gi) == 4:
            b = data[:, off:off + 8 * g]
            c[:, gi, 0::2] = b & 0xF
            c[:, gi, 1::2] = b >> 4
            off += 8 * g
        else:
            b2 = data[:, off:off + 4 * g]
            off += 4 * g
            hi = np.unpackbits(data[:, off:off + 2 * g], axis=1, bitorder="little")
            off += 2 * g
            for k in range(4):
                c[:, gi, k::4] = (b2 >> (2 * k)) & 3
            c[:, gi] |= hi << 2
    codes = c.reshape(P, lat.n_groups, PAGE, g).transpose(0, 2, 1, 3).reshape(P * PAGE, lat.r)
    m = np.asarray(meta, np.uint32).transpose(0, 2, 1).reshape(P * PAGE, lat.n_groups)
    s = (m & 0xFFFF).astype(np.uint16).view(np.float16)
    zp = (m >> 16).astype(np.uint16).view(np.float16)
    return codes, s, zp


def quantize_pack_region(z, lat: Latent):
    """Rotate, quantise and pack n pre-quantisation latents z [n, r] into ceil(n/16) pages.

    Rows past n in the last page are zero codes with zero scale/zero-point.
    """
    z = np.asarray(z, np.float32)
    n = z.shape[0]
    P = (n + PAGE - 1) // PAGE
    codes, s, zp = quantize_latent(z, lat)
    if lat.fp16:
        vv = np.zeros((P * PAGE, lat.r), np.float16)
        vv[:n] = codes
        return pack_region(vv, None, None, lat)
    cc = np.zeros((P * PAGE, lat.r), np.uint8)
    ss = np.zeros((P * PAGE, lat.n_groups), np.float16)
    zz = np.zeros((P * PAGE, lat.n_groups), np.float16)
    cc[:n], ss[:n], zz[:n] = codes, s, zp
    return pack_region(cc, ss, zz, lat)


def dequantize_region(data, meta, lat: Latent, n: int) -> np.ndarray:
    """z^ (rotated domain, fp32) of the first n tokens of packed pages."""
    codes, s, zp = unpack_region(data, meta, lat)
    if lat.fp16:
        return dequantize_codes(codes[:n], None, None, lat)
    return dequantize_codes(codes[:n], s[:n], zp[:n], lat)


# ----------------------------------------------------------------------------
# Paged latent cache  (decode dataflow steps 1-3: project, rotate, quantise, append)
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class Cache:
    cfg: Config
    k_codes: np.ndarray  # uint8  [n_pages, h_kv, key.region_bytes]
    v_codes: np.ndarray  # uint8  [n_pages, val.region_bytes]
    k_meta: np.ndarray   # uint32 [n_pages, h_kv, key.n_groups, 16]
    v_meta: np.ndarray   # uint32 [n_pages, val.n_groups, 16]


def new_cache(cfg: Config, n_pages: int) -> Cache:
    k, v = cfg.key, cfg.val
    mk = 0 if k.fp16 else k.n_groups   # fp16 latents carry no metadata
    mv = 0 if v.fp16 else v.n_groups
    if cfg.ragged:
        # ragged ranks: one flat key page per page id, the heads' regions back to back
        _, kb, km = cfg.key_layout()
        return Cache(cfg, np.zeros((n_pages, kb), np.uint8), np.zeros((n_pages, v.region_bytes), np.uint8),
                     np.zeros((n_pages, km), np.uint32), np.zeros((n_pages, mv, PAGE), np.uint32))
    return Cache(cfg,
                 np.zeros((n_pages, cfg.h_kv, k.region_bytes), np.uint8),
                 np.zeros((n_pages, v.region_bytes), np.uint8),
                 np.zeros((n_pages, cfg.h_kv, mk, PAGE), np.uint32),
                 np.zeros((n_pages, mv, PAGE), np.uint32))


def write_latents(cache: Cache, slots, z_k, z_v) -> None:
    """Quantise pre-quantisation latents and store them at physical slots.

    slots [n] = page * 16 + offset (distinct); z_k [n, h_kv, r_k]; z_v [n, R].
    Pages are unpacked, the rows replaced, and repacked; other rows keep their bits.
    """
    cfg = cache.cfg
    slots = np.asarray(slots, np.int64)
    if slots.size == 0:
        return
    pages, offs = slots // PAGE, slots % PAGE
    upages, inv = np.unique(pages, return_inverse=True)
    rows = inv * PAGE + offs
    if cfg.ragged:
        # per head: its own rank (the first r_k,h channels of z_k[:, h]) and geometry
        for h, (_, co, mo) in enumerate(cfg.key_layout()[0]):
            L = cfg.key_head(h)
            codes, s_, zp = quantize_latent(np.asarray(z_k)[:, h, :L.r], L)
            cb = cache.k_codes[upages, co:co + L.region_bytes]
            mb = cache.k_meta[upages, mo:mo + L.meta_bytes // 4].reshape(len(upages), -1, PAGE)
            cc, ss, zz = unpack_region(cb, mb, L)
            cc[rows] = codes
            if not L.fp16:
                ss[rows], zz[rows] = s_, zp
            nb, nm = pack_region(cc, ss, zz, L)
            cache.k_codes[upages, co:co + L.region_bytes] = nb
            cache.k_meta[upages, mo:mo + L.meta_bytes // 4] = nm.reshape(len(upages), -1)
        _write_values(cache, upages, rows, z_v)
        return
    if cfg.fp16_latent:
        for h in range(cfg.h_kv):
            v, _, _ = quantize_latent(np.asarray(z_k)[:, h], cfg.key)
            vv, _, _ = unpack_region(cache.k_codes[upages, h], None, cfg.key)
            vv[rows] = v
            cache.k_codes[upages, h] = pack_region(vv, None, None, cfg.key)[0]
        v, _, _ = quantize_latent(z_v, cfg.val)
        vv, _, _ = unpack_region(cache.v_codes[upages], None, cfg.val)
        vv[rows] = v
        cache.v_codes[upages] = pack_region(vv, None, None, cfg.val)[0]
        return
    for h in range(cfg.h_kv):
        codes, s, zp = quantize_latent(np.asarray(z_k)[:, h], cfg.key)
        cc, ss, zz = unpack_region(cache.k_codes[upages, h], cache.k_meta[upages, h], cfg.key)
        cc[rows], ss[rows], zz[rows] = codes, s, zp
        cache.k_codes[upages, h], cache.k_meta[upages, h] = pack_region(cc, ss, zz, cfg.key)
    codes, s, zp = quantize_latent(z_v, cfg.val)
    cc, ss, zz = unpack_region(cache.v_codes[upages], cache.v_meta[upages], cfg.val)
    cc[rows], ss[rows], zz[rows] = codes, s, zp
    cache.v_codes[upages], cache.v_meta[upages] = pack_region(cc, ss, zz, cfg.val)


def _write_values(cache: Cache, upages, rows, z_v) -> None:
    cfg = cache.cfg
    codes, s, zp = quantize_latent(z_v, cfg.val)
    cc, ss, zz = unpack_region(cache.v_codes[upages], None if cfg.val.fp16 else cache.v_meta[upages], cfg.val)
    cc[rows] = codes
    if not cfg.val.fp16:
        ss[rows], zz[rows] = s, zp
    nb, nm = pack_region(cc, ss, zz, cfg.val)
    cache.v_codes[upages] = nb
    if not cfg.val.fp16:
        cache.v_meta[upages] = nm


def pad_key_latents(cfg: Config, z) -> np.ndarray:
    """Key latents of the library's ragged layout, [n, sum_h r_k,h] (head h's
    columns at its offset), as [n, h_kv, r_k] with zeros past each head's rank."""
    z = np.asarray(z)
    out = np.zeros((z.shape[0], cfg.h_kv, cfg.r_k), z.dtype)
    for h, (col, _, _) in enumerate(cfg.key_layout()[0]):
        out[:, h, :cfg.key_rank(h)] = z[:, col:col + cfg.key_rank(h)]
    return out


def pad_key_factor(cfg: Config, B_k) -> np.ndarray:
    """B_k of the ragged layout, [sum_h r_k,h, d_h], as [h_kv, r_k, d_h] with zero
    rows past each head's rank (the padded channels then contribute nothing)."""
    B_k = np.asarray(B_k)
    out = np.zeros((cfg.h_kv, cfg.r_k, cfg.d_h), B_k.dtype)
    for h, (col, _, _) in enumerate(cfg.key_layout()[0]):
        out[h, :cfg.key_rank(h)] = B_k[col:col + cfg.key_rank(h)]
    return out


def unrotate_keys(cfg: Config, zk) -> np.ndarray:
    """Undo the key rotation of [n, h_kv, r_k] latents, each head with its own group size."""
    if not cfg.ragged:
        return unrotate_fp64(zk, cfg.key.g)
    out = np.zeros(np.shape(zk))
    for h in range(cfg.h_kv):
        L = cfg.key_head(h)
        out[:, h, :L.r] = unrotate_fp64(np.asarray(zk)[:, h, :L.r], L.g)
    return out


def append(cache: Cache, X, A_k, A_v, slots):
    """Decode dataflow steps 1-3: Z_k = X A_k, Z_v = X A_v, rotate, quantise, store.

    Returns the pre-quantisation latents (z_k [n, h_kv, r_k], z_v [n, R]) as fp32.
    """
    cfg = cache.cfg
    z_k = project(X, A_k)
    z_k = pad_key_latents(cfg, z_k) if cfg.ragged else z_k.reshape(-1, cfg.h_kv, cfg.r_k)
    z_v = project(X, A_v)
    write_latents(cache, slots, z_k, z_v)
    return z_k, z_v


def gather_sequence(cache: Cache, block_table_row, n: int):
    """Dequantised latents of positions [0, n) of one sequence (rotated domain, fp32).

    Returns (zk^ [n, h_kv, r_k], zv^ [n, R]).
    """
    cfg = cache.cfg
    P = (n + PAGE - 1) // PAGE
    pages = np.asarray(block_table_row[:P], np.int64)
    if cfg.ragged:
        zk = np.zeros((n, cfg.h_kv, cfg.r_k), np.float32)
        for h, (_, co, mo) in enumerate(cfg.key_layout()[0]):
            L = cfg.key_head(h)
            mb = cache.k_meta[pages, mo:mo + L.meta_bytes // 4].reshape(P, -1, PAGE)
            zk[:, h, :L.r] = dequantize_region(cache.k_codes[pages, co:co + L.region_bytes], mb, L, n)
        zv = dequantize_region(cache.v_codes[pages], cache.v_meta[pages], cfg.val, n)
        return zk, zv
    zk = np.stack([dequantize_region(cache.k_codes[pages, h], cache.k_meta[pages, h], cfg.key, n)
                   for h in range(cfg.h_kv)], axis=1)
    zv = dequantize_region(cache.v_codes[pages], cache.v_meta[pages], cfg.val, n)
    return zk, zv


# ----------------------------------------------------------------------------
# RoPE and attention  ([Review] section 2.3 eq. 4 scores; section 5.3 eq. 12;
# decode dataflow steps 4-8)
# ----------------------------------------------------------------------------
def rope(x, pos, base: float) -> np.ndarray:
    """Rotate-half RoPE in fp64: pairs (i, i + d/2) turned by pos * base^(-2i/d)."""
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    half = d // 2
    theta = np.float64(base) ** (-2.0 * np.arange(half, dtype=np.float64) / d)
    ang = np.asarray(pos, np.float64)[..., None] * theta
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def attend_latents(cfg: Config, z_k, z_v, q, q_pos, B_k, B_v, heads=None):
    """Attention of queries on unrotated latents (fp64).

    z_k [n, h_kv, r_k] and z_v [n, R] are the latents of positions 0..n-1;
    q [m, H, d_h] pre-RoPE queries at positions q_pos [m]; query i sees keys
    j <= q_pos[i].  Keys: k_j = z_k,j B_k,h, RoPE'd at position j (pre-RoPE latent
    keys, [Review] section 5.3).  Values: the stacked probabilities multiply the
    shared joint latent, o_lat,h = p_h Z_V, then o_h = o_lat,h B_v[:, kv(h)]
    ([Review] eq. 12 and the stacked P Z_V product).
    Returns o [m, len(heads), d_h] (fp64).
    """
    z_k = np.asarray(z_k, np.float64)
    z_v = np.asarray(z_v, np.float64)
    q = np.asarray(q, np.float64)
    B_k = np.asarray(B_k, np.float64)
    B_v = np.asarray(B_v, np.float64)
    n = z_k.shape[0]
    d = cfg.d_h
    heads = list(range(cfg.H)) if heads is None else list(heads)
    q_pos = np.asarray(q_pos, np.int64)
    pos = np.arange(n)
    mask = pos[None, :] <= q_pos[:, None]                     # [m, n]
    out = np.empty((q.shape[0], len(heads), d))
    krope = {}
    for oi, h in enumerate(heads):
        kv = h // cfg.group
        if kv not in krope:
            krope[kv] = rope(z_k[:, kv] @ B_k[kv], pos, cfg.rope_base)   # [n, d]
        qr = rope(q[:, h], q_pos, cfg.rope_base)                        # [m, d]
        sc = (qr @ krope[kv].T) / np.sqrt(d)
        sc = np.where(mask, sc, -np.inf)
        sc = sc - sc.max(axis=1, keepdims=True)
        p = np.exp(sc)
        p /= p.sum(axis=1, keepdims=True)
        o_lat = p @ z_v                                                  # [m, R]
        out[:, oi] = o_lat @ B_v[:, kv * d:(kv + 1) * d]
    return out


def decode(cache: Cache, q, B_k, B_v, block_table, seq_lens, seqs=None, heads=None):
    """starkv_decode_attn: each sequence's single query, at position seq_len - 1,
    attends to positions [0, seq_len) of the quantised cache.  A sequence with
    no tokens (seq_len 0) has nothing to attend to; the boundary defines its
    output row as zeros.

    Returns o [B, H, d_h] fp64 (NaN where not requested by ``seqs``/``heads``).
    """
    cfg = cache.cfg
    q = np.asarray(q)
    Bn = q.shape[0]
    out = np.full((Bn, cfg.H, cfg.d_h), np.nan)
    heads = list(range(cfg.H)) if heads is None else list(heads)
    for b in (range(Bn) if seqs is None else seqs):
        n = int(seq_lens[b])
        if n == 0:
            out[b, heads] = 0.0
            continue
        zk, zv = gather_sequence(cache, block_table[b], n)
        zk = unrotate_keys(cfg, zk)
        zv = unrotate_fp64(zv, cfg.val.g)
        out[b, heads] = attend_latents(cfg, zk, zv, q[b:b + 1], [n - 1], B_k, B_v, heads)[0]
    return out


def decode_out(cache: Cache, q, B_k, B_v, W_o, block_table, seq_lens):
    """starkv_decode_attn_out: the attention block's output, decode dataflow
    steps 7-8 ([Review] Algorithm 2: apply the head-specific value/output
    factors, sum the head contributions; eq. 12):
    y[b] = sum_h o_h[b] W_o[h d_h : (h + 1) d_h, :] with o from ``decode``.
    W_o: [H d_h, model_dim].  Returns y [B, model_dim] (fp64)."""
    cfg = cache.cfg
    o = decode(cache, q, B_k, B_v, block_table, seq_lens)
    W_o = np.asarray(W_o, np.float64)
    return o.reshape(o.shape[0], cfg.H * cfg.d_h) @ W_o


def decode_slice(cache: Cache, q, B_k, B_v, block_table, seq_lens, key_pos0, q_pos, heads=None):
    """starkv_decode_attn_slice: sequence b's cache holds one slice of its context,
    seq_lens[b] tokens at positions key_pos0[b] .. key_pos0[b] + seq_lens[b] - 1
    (block-table row from local index 0), and its query sits at q_pos[b].  The
    query attends to the slice alone ([CaliDrop] attention decomposition theorem,
    eq. 1: partials of disjoint key subsets merge exactly).

    Returns (o [B, H, d_h] normalised within the slice, m [B, H], l [B, H]) in
    natural-log units: m = max_j s_j, l = sum_j e^(s_j - m); an empty slice gives
    (0, -inf, 0).  NaN where not requested by ``heads``.
    """
    cfg = cache.cfg
    q = np.asarray(q)
    Bn = q.shape[0]
    d = cfg.d_h
    heads = list(range(cfg.H)) if heads is None else list(heads)
    o = np.full((Bn, cfg.H, d), np.nan)
    m = np.full((Bn, cfg.H), np.nan)
    l = np.full((Bn, cfg.H), np.nan)
    B_k = np.asarray(B_k, np.float64)
    B_v = np.asarray(B_v, np.float64)
    for b in range(Bn):
        n = int(seq_lens[b])
        if n == 0:
            o[b, heads], m[b, heads], l[b, heads] = 0.0, -np.inf, 0.0
            continue
        zk, zv = gather_sequence(cache, block_table[b], n)
        zk = unrotate_keys(cfg, zk)
        zv = unrotate_fp64(zv, cfg.val.g)
        pos = int(key_pos0[b]) + np.arange(n)
        for h in heads:
            kv = h // cfg.group
            k = rope(zk[:, kv] @ B_k[kv], pos, cfg.rope_base)
            qr = rope(np.asarray(q[b, h], np.float64), int(q_pos[b]), cfg.rope_base)
            s = (k @ qr) / np.sqrt(d)
            mb, lb, acc = partial_softmax(s, zv)
            o[b, h] = (acc / lb) @ B_v[:, kv * d:(kv + 1) * d]
            m[b, h], l[b, h] = mb, lb
    return o, m, l


def merge_slices(o_parts, m_parts, l_parts):
    """Combine slice results of the same queries (the partition identity):
    o = sum_r e^(m_r - M) l_r o_r / sum_r e^(m_r - M) l_r, M = max_r m_r over the
    non-empty slices.  Inputs stacked on a leading slice axis: o [n, ..., d],
    m and l [n, ...].  All slices empty: zeros."""
    o_parts = np.asarray(o_parts, np.float64)
    m_parts = np.asarray(m_parts, np.float64)
    l_parts = np.asarray(l_parts, np.float64)
    live = l_parts > 0
    M = np.where(live, m_parts, -np.inf).max(axis=0)
    w = np.where(live, np.exp(np.where(live, m_parts, 0.0) - np.where(np.isfinite(M), M, 0.0)) * l_parts, 0.0)
    den = w.sum(axis=0)
    num = (w[..., None] * o_parts).sum(axis=0)
    return np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)


def prefill(cache: Cache, q, cu_q, B_k, B_v, block_table, seq_lens, select=None, heads=None):
    """starkv_prefill_attn: query i of sequence b (cu_q[b] <= row < cu_q[b+1]) sits at
    position seq_len_b - n_b + i and attends causally to positions <= its own.

    select: optional {b: [query indices within the sequence]}.
    Returns o [Nq, H, d_h] fp64 (NaN where not requested).
    """
    cfg = cache.cfg
    q = np.asarray(q)
    out = np.full((q.shape[0], cfg.H, cfg.d_h), np.nan)
    heads = list(range(cfg.H)) if heads is None else list(heads)
    Bn = len(cu_q) - 1
    for b in range(Bn):
        nb = int(cu_q[b + 1] - cu_q[b])
        if nb == 0 or (select is not None and b not in select):
            continue
        idx = np.arange(nb) if select is None else np.asarray(select[b], np.int64)
        if idx.size == 0:
            continue
        n = int(seq_lens[b])
        zk, zv = gather_sequence(cache, block_table[b], n)
        zk = unrotate_keys(cfg, zk)
        zv = unrotate_fp64(zv, cfg.val.g)
        rows = int(cu_q[b]) + idx
        out[np.ix_(rows, heads)] = attend_latents(cfg, zk, zv, q[rows], n - nb + idx, B_k, B_v, heads)
    return out


# ----------------------------------------------------------------------------
# Split-K merge  ([CaliDrop] attention decomposition theorem, eq. 1)
# ----------------------------------------------------------------------------
def partial_softmax(scores, values):
    """(m, l, acc) of one key subset: m = max s, l = sum e^(s-m), acc = sum e^(s-m) v."""
    scores = np.asarray(scores, np.float64)
    values = np.asarray(values, np.float64)
    if scores.size == 0:
        return -np.inf, 0.0, np.zeros(values.shape[1:])
    m = scores.max()
    e = np.exp(scores - m)
    return m, e.sum(), e @ values


def lse_merge(parts):
    """Merge subset partials: weights alpha_i = each subset's share of sum e^s."""
    m = max(p[0] for p in parts)
    w = [np.exp(p[0] - m) if np.isfinite(p[0]) else 0.0 for p in parts]
    l = sum(wi * p[1] for wi, p in zip(w, parts))
    acc = sum(wi * p[2] for wi, p in zip(w, parts))
    return acc / l


# ----------------------------------------------------------------------------
# Byte accounting  ([Review] eq. 1, 14, 15, 16)
# ----------------------------------------------------------------------------
def eq1_dense_payload_bytes(B, T, L, h_kv, d_h, bits) -> float:
    """M_KV = 2 B T L h_kv d_h b / 8 (keys and values; KV heads, not query heads)."""
    return 2 * B * T * L * h_kv * d_h * bits / 8


def eq14_mean_bits(top_fraction, top_bits=4, bottom_bits=3) -> float:
    return top_fraction * top_bits + (1 - top_fraction) * bottom_bits


def eq14_payload_compression(rho, mean_bits) -> float:
    """C_payload = 16 / (rho b-bar) against an fp16 payload."""
    return 16.0 / (rho * mean_bits)


def eq15_latent_payload_bytes(B, T, mean_bits, key_ranks_per_layer, value_rank_per_layer) -> float:
    """M_latent payload = (B T b-bar / 8) sum_l (sum_h r^K_{l,h} + R^V_l)."""
    tot = sum(sum(kr) + rv for kr, rv in zip(key_ranks_per_layer, value_rank_per_layer))
    return B * T * mean_bits / 8 * tot


def eq16_retained_fraction(L=32, exempt=3, compressed_fraction=0.25 * 3.2 / 16) -> float:
    return exempt / L + (L - exempt) / L * compressed_fraction


def layout_sizes(cfg: Config, n_pages: int) -> dict:
    """Bytes of the four cache pools for n_pages pages (the packed layout above)."""
    k, v = cfg.key, cfg.val
    _, kb, km = cfg.key_layout()
    return dict(k_codes=n_pages * kb,
                v_codes=n_pages * v.region_bytes,
                k_meta=n_pages * km * 4,
                v_meta=n_pages * v.meta_bytes)


def cache_bytes_per_token(cfg: Config) -> float:
    return sum(layout_sizes(cfg, 1).values()) / PAGE


def payload_bytes_per_token(cfg: Config) -> float:
    return (sum(cfg.key_head(h).payload_bytes for h in range(cfg.h_kv)) + cfg.val.payload_bytes) / PAGE
