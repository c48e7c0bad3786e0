"""Planted mistakes: the oracle's pins must catch plausible errors in it.

Each case replaces one oracle function by a copy of it with a single planted
mistake (a flipped sign, a transposed pairing, a dropped term or weight, an
off-by-one position, a swapped bit field), runs the pins that guard that
function, and requires at least one of them to fail.  The same copies with no
mistake planted pass the same pins, so every failure comes from the plant.
Everything here runs in the oracle, on the CPU; nothing touches the library.
"""
import numpy as np
import pytest

import oracle as O
import oracle.starkv_oracle as OM
import test_oracle_attention as TA
import test_oracle_bytes as TB
import test_oracle_quant as TQ


# ----------------------------------------------------------------------------
# copies of oracle functions with one knob per plausible mistake
# (defaults reproduce the oracle exactly)
# ----------------------------------------------------------------------------
def rope_k(sign=1.0, pairing="half", expo=2.0, shift=0.0):
    def rope(x, pos, base):
        x = np.asarray(x, np.float64)
        d = x.shape[-1]
        half = d // 2
        theta = np.float64(base) ** (-expo * np.arange(half, dtype=np.float64) / d)
        ang = (np.asarray(pos, np.float64)[..., None] + shift) * theta
        c, s = np.cos(ang), sign * np.sin(ang)
        if pairing == "half":
            a, b = x[..., :half], x[..., half:]
            return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)
        out = np.empty_like(x)
        a, b = x[..., 0::2], x[..., 1::2]
        out[..., 0::2], out[..., 1::2] = a * c - b * s, b * c + a * s
        return out
    return rope


def hadamard_k(normalise=True, lower_sign=False):
    def hadamard_fp64(g):
        h = np.ones((1, 1))
        while h.shape[0] < g:
            h = np.block([[h, h], [-h, h]]) if lower_sign else np.block([[h, h], [h, -h]])
        return h / np.sqrt(g) if normalise else h
    return hadamard_fp64


def rotate_k(flip=False, scale=True):
    def rotate_fl32(z, g):
        z = np.asarray(z, np.float32)
        shp = z.shape
        x = z.reshape(-1, shp[-1] // g, g)
        h = 1
        while h < g:
            y = x.reshape(x.shape[0], x.shape[1], g // (2 * h), 2, h)
            a, b = y[..., 0, :], y[..., 1, :]
            x = np.stack([a + b, b - a if flip else a - b], axis=-2).reshape(x.shape[0], x.shape[1], g)
            h *= 2
        return (x * OM.inv_sqrt_fl32(g) if scale else x).reshape(shp)
    return rotate_fl32


def unrotate_k(identity=False):
    def unrotate_fp64(zr, g):
        zr = np.asarray(zr, np.float64)
        if identity:
            return zr.copy()
        shp = zr.shape
        return (zr.reshape(-1, shp[-1] // g, g) @ OM.hadamard_fp64(g)).reshape(shp)
    return unrotate_fp64


def quantize_k(levels_pow2=False, rounding="rint", zero="min"):
    def quantize_groups(zr, bits):
        zr = np.asarray(zr, np.float32)
        mn, mx = zr.min(axis=-1), zr.max(axis=-1)
        qmax = np.float32(2 ** bits - 1)
        div = np.float32(2 ** bits) if levels_pow2 else qmax
        with np.errstate(over="ignore"):
            s = ((mx - mn) / div).astype(np.float16)
            zp = (mn if zero == "min" else mx).astype(np.float16)
        if not (np.isfinite(s).all() and np.isfinite(zp).all()):
            raise OM.QuantError("fp16 scale or zero-point overflow")
        sf = s.astype(np.float32)[..., None]
        zf = zp.astype(np.float32)[..., None]
        with np.errstate(divide="ignore", invalid="ignore"):
            qv = (zr - zf) / sf
        r = np.rint(qv) if rounding == "rint" else np.floor(qv)
        code = np.where(sf == 0, np.float32(0), np.clip(r, np.float32(0), qmax))
        return code.astype(np.uint8), s, zp
    return quantize_groups


def dequantize_k(zp_sign=1.0, half_step=False):
    def dequantize_codes(codes, s, zp, lat):
        n = codes.shape[0]
        c = codes.reshape(n, lat.n_groups, lat.g).astype(np.float32)
        if half_step:
            c = c + np.float32(0.5)
        zh = c * s.astype(np.float32)[..., None] + np.float32(zp_sign) * zp.astype(np.float32)[..., None]
        return zh.reshape(n, lat.r)
    return dequantize_codes


def quantize_latent_k(all_bits=None, top_shift=0, fp16_unrotated=False):
    def quantize_latent(z, lat):
        z = np.asarray(z, np.float32)
        n = z.shape[0]
        if lat.fp16:
            v = (z if fp16_unrotated else OM.rotate_fl32(z, lat.g)).astype(np.float16)
            return v, None, None
        zr = OM.rotate_fl32(z, lat.g).reshape(n, lat.n_groups, lat.g)
        codes = np.empty((n, lat.n_groups, lat.g), np.uint8)
        s = np.empty((n, lat.n_groups), np.float16)
        zp = np.empty((n, lat.n_groups), np.float16)
        t = min(max(lat.n_top_groups + top_shift, 0), lat.n_groups)
        if all_bits is not None:
            t = lat.n_groups if all_bits == 4 else 0
        if t:
            codes[:, :t], s[:, :t], zp[:, :t] = OM.quantize_groups(zr[:, :t], 4)
        if t < lat.n_groups:
            codes[:, t:], s[:, t:], zp[:, t:] = OM.quantize_groups(zr[:, t:], 3)
        return codes.reshape(n, lat.r), s, zp
    return quantize_latent


def pack_k(hi_first=False, planes_swapped=False, meta_swapped=False, fp16_channel_major=False):
    def pack_region(codes, s, zp, lat):
        if lat.fp16:
            v = np.asarray(codes, np.float16)
            P = v.shape[0] // OM.PAGE
            tiles = v.reshape(P, OM.PAGE, lat.n_groups, lat.g).transpose(0, 2, 1, 3)
            if fp16_channel_major:
                tiles = tiles.transpose(0, 1, 3, 2)
            return (np.ascontiguousarray(tiles).view(np.uint8).reshape(P, lat.region_bytes).copy(),
                    np.zeros((P, 0, OM.PAGE), np.uint32))
        codes = np.asarray(codes, np.uint8)
        P = codes.shape[0] // OM.PAGE
        g = lat.g
        c = codes.reshape(P, OM.PAGE, lat.n_groups, g).transpose(0, 2, 1, 3).reshape(P, lat.n_groups, OM.PAGE * g)
        out = np.zeros((P, lat.region_bytes), np.uint8)
        off = 0
        for gi in range(lat.n_groups):
            tile = c[:, gi]
            if lat.group_bits(gi) == 4:
                lo, hi = (tile[:, 1::2], tile[:, 0::2]) if hi_first else (tile[:, 0::2], tile[:, 1::2])
                out[:, off:off + 8 * g] = (lo & 0xF) | ((hi & 0xF) << 4)
                off += 8 * g
            else:
                two = tile & 3
                p2 = two[:, 0::4] | (two[:, 1::4] << 2) | (two[:, 2::4] << 4) | (two[:, 3::4] << 6)
                p1 = np.packbits((tile >> 2) & 1, axis=1, bitorder="little")
                for plane in ((p1, p2) if planes_swapped else (p2, p1)):
                    out[:, off:off + plane.shape[1]] = plane
                    off += plane.shape[1]
        s16 = np.asarray(s, np.float16).view(np.uint16).astype(np.uint32)
        z16 = np.asarray(zp, np.float16).view(np.uint16).astype(np.uint32)
        meta = (z16 | (s16 << 16)) if meta_swapped else (s16 | (z16 << 16))
        return out, meta.reshape(P, OM.PAGE, lat.n_groups).transpose(0, 2, 1).copy()
    return pack_region


def write_k(drop_offsets=False):
    real = OM.write_latents

    def write_latents(cache, slots, z_k, z_v):
        cfg = cache.cfg
        if cfg.ragged:
            return real(cache, slots, z_k, z_v)
        slots = np.asarray(slots, np.int64)
        if slots.size == 0:
            return
        pages, offs = slots // OM.PAGE, slots % OM.PAGE
        upages, inv = np.unique(pages, return_inverse=True)
        rows = inv * OM.PAGE + (0 if drop_offsets else offs)
        for h in range(cfg.h_kv):
            codes, s, zp = OM.quantize_latent(np.asarray(z_k)[:, h], cfg.key)
            cc, ss, zz = OM.unpack_region(cache.k_codes[upages, h], cache.k_meta[upages, h], cfg.key)
            cc[rows], ss[rows], zz[rows] = codes, s, zp
            cache.k_codes[upages, h], cache.k_meta[upages, h] = OM.pack_region(cc, ss, zz, cfg.key)
        codes, s, zp = OM.quantize_latent(z_v, cfg.val)
        cc, ss, zz = OM.unpack_region(cache.v_codes[upages], cache.v_meta[upages], cfg.val)
        cc[rows], ss[rows], zz[rows] = codes, s, zp
        cache.v_codes[upages], cache.v_meta[upages] = OM.pack_region(cc, ss, zz, cfg.val)
    return write_latents


def gather_k(ignore_table=False):
    def gather_sequence(cache, block_table_row, n):
        cfg = cache.cfg
        P = (n + OM.PAGE - 1) // OM.PAGE
        pages = np.arange(P) if ignore_table else np.asarray(block_table_row[:P], np.int64)
        zk = np.stack([OM.dequantize_region(cache.k_codes[pages, h], cache.k_meta[pages, h], cfg.key, n)
                       for h in range(cfg.h_kv)], axis=1)
        zv = OM.dequantize_region(cache.v_codes[pages], cache.v_meta[pages], cfg.val, n)
        return zk, zv
    return gather_sequence


def attend_k(scale_pow=0.5, kv_of="div", strict=False, v_head0=False, qshift=0):
    def attend_latents(cfg, z_k, z_v, q, q_pos, B_k, B_v, heads=None):
        z_k, z_v, q = (np.asarray(a, np.float64) for a in (z_k, z_v, q))
        B_k, B_v = np.asarray(B_k, np.float64), np.asarray(B_v, np.float64)
        n, d = z_k.shape[0], cfg.d_h
        heads = list(range(cfg.H)) if heads is None else list(heads)
        q_pos = np.asarray(q_pos, np.int64) + qshift
        pos = np.arange(n)
        mask = pos[None, :] < q_pos[:, None] if strict else pos[None, :] <= q_pos[:, None]
        out = np.empty((q.shape[0], len(heads), d))
        for oi, h in enumerate(heads):
            kv = h // cfg.group if kv_of == "div" else h % cfg.h_kv
            k = OM.rope(z_k[:, kv] @ B_k[kv], pos, cfg.rope_base)
            qr = OM.rope(q[:, h], q_pos, cfg.rope_base)
            sc = np.where(mask, (qr @ k.T) / float(d) ** scale_pow, -np.inf)
            with np.errstate(invalid="ignore"):
                p = np.exp(sc - sc.max(axis=1, keepdims=True))
                p /= p.sum(axis=1, keepdims=True)
            vk = 0 if v_head0 else kv
            out[:, oi] = (p @ z_v) @ B_v[:, vk * d:(vk + 1) * d]
        return out
    return attend_latents


def partial_k(unweighted_acc=False):
    def partial_softmax(scores, values):
        scores, values = np.asarray(scores, np.float64), np.asarray(values, np.float64)
        if scores.size == 0:
            return -np.inf, 0.0, np.zeros(values.shape[1:])
        m = scores.max()
        e = np.exp(scores - m)
        return m, e.sum(), (values.sum(0) if unweighted_acc else e @ values)
    return partial_softmax


def merge_k(weight_l=True):
    def lse_merge(parts):
        m = max(p[0] for p in parts)
        w = [np.exp(p[0] - m) if np.isfinite(p[0]) else 0.0 for p in parts]
        l = sum((wi if weight_l else 1.0) * p[1] for wi, p in zip(w, parts))
        return sum(wi * p[2] for wi, p in zip(w, parts)) / l
    return lse_merge


def project_k(fp32_accumulate=False, keep_fp64=False):
    def project(X, A):
        if fp32_accumulate:
            X32, A32 = np.asarray(X, np.float32), np.asarray(A, np.float32)
            out = np.zeros((X32.shape[0], A32.shape[1]), np.float32)
            for k in range(X32.shape[1]):
                out += X32[:, k:k + 1] * A32[k:k + 1, :]
            return out
        prod = np.asarray(X, np.float64) @ np.asarray(A, np.float64)
        return prod if keep_fp64 else prod.astype(np.float32)
    return project


def decode_slice_k(ignore_pos0=False, q_at_end_of_slice=False):
    def decode_slice(cache, q, B_k, B_v, block_table, seq_lens, key_pos0, q_pos, heads=None):
        cfg = cache.cfg
        q = np.asarray(q)
        Bn, d = q.shape[0], cfg.d_h
        heads = list(range(cfg.H)) if heads is None else list(heads)
        o = np.full((Bn, cfg.H, d), np.nan)
        m = np.full((Bn, cfg.H), np.nan)
        l = np.full((Bn, cfg.H), np.nan)
        B_k, B_v = np.asarray(B_k, np.float64), np.asarray(B_v, np.float64)
        for b in range(Bn):
            n = int(seq_lens[b])
            if n == 0:
                o[b, heads], m[b, heads], l[b, heads] = 0.0, -np.inf, 0.0
                continue
            zk, zv = OM.gather_sequence(cache, block_table[b], n)
            zk, zv = OM.unrotate_fp64(zk, cfg.key.g), OM.unrotate_fp64(zv, cfg.val.g)
            pos = (0 if ignore_pos0 else int(key_pos0[b])) + np.arange(n)
            qp = (int(key_pos0[b]) + n - 1) if q_at_end_of_slice else int(q_pos[b])
            for h in heads:
                kv = h // cfg.group
                k = OM.rope(zk[:, kv] @ B_k[kv], pos, cfg.rope_base)
                qr = OM.rope(np.asarray(q[b, h], np.float64), qp, cfg.rope_base)
                mb, lb, acc = OM.partial_softmax((k @ qr) / np.sqrt(d), zv)
                o[b, h] = (acc / lb) @ B_v[:, kv * d:(kv + 1) * d]
                m[b, h], l[b, h] = mb, lb
        return o, m, l
    return decode_slice


def merge_slices_k(drop_l=False, flip=False):
    def merge_slices(o_parts, m_parts, l_parts):
        o_parts, m_parts, l_parts = (np.asarray(a, np.float64) for a in (o_parts, m_parts, l_parts))
        live = l_parts > 0
        M = np.where(live, m_parts, -np.inf).max(axis=0)
        e = np.where(live, m_parts, 0.0) - np.where(np.isfinite(M), M, 0.0)
        w = np.where(live, np.exp(-e if flip else e) * (1.0 if drop_l else l_parts), 0.0)
        den = w.sum(axis=0)
        num = (w[..., None] * o_parts).sum(axis=0)
        return np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)
    return merge_slices


def decode_out_k(kv_rows=False):
    def decode_out(cache, q, B_k, B_v, W_o, block_table, seq_lens):
        cfg = cache.cfg
        o = OM.decode(cache, q, B_k, B_v, block_table, seq_lens)
        W_o = np.asarray(W_o, np.float64)
        if not kv_rows:
            return o.reshape(o.shape[0], cfg.H * cfg.d_h) @ W_o
        d = cfg.d_h
        return sum(o[:, h] @ W_o[(h // cfg.group) * d:(h // cfg.group + 1) * d] for h in range(cfg.H))
    return decode_out


def write_ragged_k(reverse_heads=False):
    real = OM.write_latents

    def write_latents(cache, slots, z_k, z_v):
        cfg = cache.cfg
        if not cfg.ragged:
            return real(cache, slots, z_k, z_v)
        slots = np.asarray(slots, np.int64)
        pages, offs = slots // OM.PAGE, slots % OM.PAGE
        upages, inv = np.unique(pages, return_inverse=True)
        rows = inv * OM.PAGE + offs
        rev = {}
        if reverse_heads:   # the heads' regions placed in reverse head order
            co_, mo_ = 0, 0
            for h in reversed(range(cfg.h_kv)):
                L = cfg.key_head(h)
                rev[h] = (co_, mo_)
                co_, mo_ = co_ + L.region_bytes, mo_ + L.meta_bytes // 4
        for h, (_, co, mo) in enumerate(cfg.key_layout()[0]):
            L = cfg.key_head(h)
            if reverse_heads:
                co, mo = rev[h]
            codes, s_, zp = OM.quantize_latent(np.asarray(z_k)[:, h, :L.r], L)
            cb = cache.k_codes[upages, co:co + L.region_bytes]
            mb = cache.k_meta[upages, mo:mo + L.meta_bytes // 4].reshape(len(upages), -1, OM.PAGE)
            cc, ss, zz = OM.unpack_region(cb, mb, L)
            cc[rows], ss[rows], zz[rows] = codes, s_, zp
            nb, nm = OM.pack_region(cc, ss, zz, L)
            cache.k_codes[upages, co:co + L.region_bytes] = nb[:, :cb.shape[1]]
            cache.k_meta[upages, mo:mo + L.meta_bytes // 4] = nm.reshape(len(upages), -1)[:, :mb.shape[1] * OM.PAGE]
        OM._write_values(cache, upages, rows, z_v)
    return write_latents


def unrotate_keys_k(widest_group=False):
    def unrotate_keys(cfg, zk):
        if not cfg.ragged:
            return OM.unrotate_fp64(zk, cfg.key.g)
        out = np.zeros(np.shape(zk))
        for h in range(cfg.h_kv):
            L = cfg.key_head(h)
            g = cfg.key.g if widest_group else L.g
            out[:, h, :L.r] = OM.unrotate_fp64(np.asarray(zk)[:, h, :L.r], g)
        return out
    return unrotate_keys


def prefill_k(shift=0):
    def prefill(cache, q, cu_q, B_k, B_v, block_table, seq_lens, select=None, heads=None):
        cfg = cache.cfg
        q = np.asarray(q)
        out = np.full((q.shape[0], cfg.H, cfg.d_h), np.nan)
        heads = list(range(cfg.H)) if heads is None else list(heads)
        for b in range(len(cu_q) - 1):
            nb = int(cu_q[b + 1] - cu_q[b])
            if nb == 0 or (select is not None and b not in select):
                continue
            idx = np.arange(nb) if select is None else np.asarray(select[b], np.int64)
            if idx.size == 0:
                continue
            n = int(seq_lens[b])
            zk, zv = OM.gather_sequence(cache, block_table[b], n)
            zk, zv = OM.unrotate_fp64(zk, cfg.key.g), OM.unrotate_fp64(zv, cfg.val.g)
            rows = int(cu_q[b]) + idx
            out[np.ix_(rows, heads)] = OM.attend_latents(cfg, zk, zv, q[rows], n - nb + idx + shift, B_k, B_v, heads)
        return out
    return prefill


def eq14_k(swap=False):
    def eq14_mean_bits(top_fraction, top_bits=4, bottom_bits=3):
        if swap:
            top_bits, bottom_bits = bottom_bits, top_bits
        return top_fraction * top_bits + (1 - top_fraction) * bottom_bits
    return eq14_mean_bits


def eq16_k(drop_exempt=False):
    def eq16_retained_fraction(L=32, exempt=3, compressed_fraction=0.25 * 3.2 / 16):
        return (0.0 if drop_exempt else exempt / L) + (L - exempt) / L * compressed_fraction
    return eq16_retained_fraction


# ----------------------------------------------------------------------------
# the pins that guard each function
# ----------------------------------------------------------------------------
PINS = {
    "rope": [lambda: TA.test_rope_matches_transformers(128, 1e4),
             lambda: TA.test_reassociated_equals_materialised(4, 4)],
    "hadamard_fp64": [lambda: TQ.test_hadamard_matches_scipy(8),
                      lambda: TQ.test_fwht_within_fp32_bound_of_matrix_product(8)],
    "rotate_fl32": [lambda: TQ.test_fwht_within_fp32_bound_of_matrix_product(8)],
    "unrotate_fp64": [lambda: TQ.test_fwht_within_fp32_bound_of_matrix_product(8),
                      lambda: TA.test_full_rank_latents_reproduce_dense_attention(True)],
    "quantize_groups": [lambda: TQ.test_grid_values_round_trip(4),
                        lambda: TQ.test_codes_are_nearest_grid_point_bruteforce(3),
                        lambda: TQ.test_quantisation_error_bound(4)],
    "dequantize_codes": [lambda: TA.test_quantised_attention_close_to_unquantised(),
                         lambda: TQ.test_grid_values_round_trip(4),
                         lambda: TQ.test_constant_group_has_zero_scale()],
    "quantize_latent": [lambda: TQ.test_quantize_latent_bit_width_per_group(64),
                        lambda: TQ.test_quantize_latent_bit_width_per_group(32),
                        lambda: TQ.test_quantize_latent_scale_per_group_on_hand_built_input(),
                        lambda: TA.test_fp16_variant_attention_close_to_unquantised(0)],
    "pack_region": [lambda: TQ.test_pack_matches_hand_derived_bytes(),
                    lambda: TQ.test_pack_unpack_exhaustive(32, 0.25),
                    lambda: TQ.test_fp16_variant_page_bytes_by_hand()],
    "write_latents": [lambda: TQ.test_write_latents_partial_pages_keep_other_rows(),
                      lambda: TB.test_ragged_pages_hold_each_heads_own_codes()],
    "unrotate_keys": [lambda: TA.test_ragged_ranks_decode_against_materialised()],
    "gather_sequence": [lambda: TA.test_decode_through_paged_cache_equals_direct()],
    "attend_latents": [lambda: TA.test_reassociated_equals_materialised(8, 2),
                       lambda: TA.test_decode_through_paged_cache_equals_direct()],
    "partial_softmax": [lambda: TA.test_partition_identity_merge()],
    "lse_merge": [lambda: TA.test_partition_identity_merge()],
    "project": [lambda: TQ.test_projection_is_the_correctly_rounded_product()],
    "prefill": [lambda: TA.test_prefill_is_causal_decode_per_query()],
    "decode_slice": [lambda: TA.test_slices_merge_to_the_whole_decode(0),
                     lambda: TA.test_slice_statistics_against_materialised_scores()],
    "merge_slices": [lambda: TA.test_slices_merge_to_the_whole_decode(0)],
    "decode_out": [lambda: TA.test_output_projection_equals_fused_factor_and_dense(8, 2)],
    "eq14_mean_bits": [lambda: TB.test_eq14_printed_values()],
    "eq16_retained_fraction": [lambda: TB.test_eq16_printed_values()],
}

FAITHFUL = {
    "rope": rope_k(), "hadamard_fp64": hadamard_k(), "rotate_fl32": rotate_k(),
    "unrotate_fp64": unrotate_k(), "quantize_groups": quantize_k(), "dequantize_codes": dequantize_k(),
    "quantize_latent": quantize_latent_k(),
    "pack_region": pack_k(), "write_latents": write_ragged_k(), "unrotate_keys": unrotate_keys_k(), "gather_sequence": gather_k(),
    "attend_latents": attend_k(), "partial_softmax": partial_k(), "lse_merge": merge_k(),
    "eq14_mean_bits": eq14_k(), "eq16_retained_fraction": eq16_k(), "project": project_k(), "prefill": prefill_k(),
    "decode_slice": decode_slice_k(), "merge_slices": merge_slices_k(), "decode_out": decode_out_k(),
}

PLANTS = {
    "rope turns the other way": ("rope", rope_k(sign=-1.0)),
    "rope pairs neighbours (2i, 2i+1) instead of halves": ("rope", rope_k(pairing="pairs")),
    "rope frequency exponent i/d instead of 2i/d": ("rope", rope_k(expo=1.0)),
    "rope position off by one": ("rope", rope_k(shift=1.0)),
    "hadamard not normalised": ("hadamard_fp64", hadamard_k(normalise=False)),
    "hadamard sign on the wrong block": ("hadamard_fp64", hadamard_k(lower_sign=True)),
    "butterfly difference b - a": ("rotate_fl32", rotate_k(flip=True)),
    "butterfly scale 1/sqrt(g) dropped": ("rotate_fl32", rotate_k(scale=False)),
    "inverse rotation skipped": ("unrotate_fp64", unrotate_k(identity=True)),
    "scale divides by 2^b, not 2^b - 1": ("quantize_groups", quantize_k(levels_pow2=True)),
    "codes truncated, not rounded": ("quantize_groups", quantize_k(rounding="floor")),
    "zero point at the group maximum": ("quantize_groups", quantize_k(zero="max")),
    "dequant subtracts the zero point": ("dequantize_codes", dequantize_k(zp_sign=-1.0)),
    "dequant adds half a step": ("dequantize_codes", dequantize_k(half_step=True)),
    "every group quantised at 3 bits": ("quantize_latent", quantize_latent_k(all_bits=3)),
    "every group quantised at 4 bits": ("quantize_latent", quantize_latent_k(all_bits=4)),
    "4-bit block one group too wide": ("quantize_latent", quantize_latent_k(top_shift=1)),
    "4-bit block one group too narrow": ("quantize_latent", quantize_latent_k(top_shift=-1)),
    "fp16 variant stores the unrotated latent": ("quantize_latent", quantize_latent_k(fp16_unrotated=True)),
    "fp16 variant tiles channel-major": ("pack_region", pack_k(fp16_channel_major=True)),
    "4-bit tile: high nibble first": ("pack_region", pack_k(hi_first=True)),
    "3-bit tile: 1-bit plane before 2-bit plane": ("pack_region", pack_k(planes_swapped=True)),
    "metadata: zero in the low half": ("pack_region", pack_k(meta_swapped=True)),
    "append drops the in-page offset": ("write_latents", write_k(drop_offsets=True)),
    "ragged heads stored in reverse order": ("write_latents", write_ragged_k(reverse_heads=True)),
    "ragged heads unrotated with the widest group": ("unrotate_keys", unrotate_keys_k(widest_group=True)),
    "gather ignores the block table": ("gather_sequence", gather_k(ignore_table=True)),
    "scores scaled by 1/d, not 1/sqrt(d)": ("attend_latents", attend_k(scale_pow=1.0)),
    "GQA head maps to h mod h_kv": ("attend_latents", attend_k(kv_of="mod")),
    "query does not see its own position": ("attend_latents", attend_k(strict=True)),
    "every head projects through KV head 0's B_v": ("attend_latents", attend_k(v_head0=True)),
    "query position one past seq_len - 1": ("attend_latents", attend_k(qshift=1)),
    "split partial sums values without weights": ("partial_softmax", partial_k(unweighted_acc=True)),
    "split merge leaves l unweighted": ("lse_merge", merge_k(weight_l=False)),
    "projection accumulated in fp32": ("project", project_k(fp32_accumulate=True)),
    "projection left in fp64": ("project", project_k(keep_fp64=True)),
    "prefill queries one position late": ("prefill", prefill_k(shift=1)),
    "slice keys RoPE'd at local positions": ("decode_slice", decode_slice_k(ignore_pos0=True)),
    "slice query at the slice's last position": ("decode_slice", decode_slice_k(q_at_end_of_slice=True)),
    "slice merge without the slice sums": ("merge_slices", merge_slices_k(drop_l=True)),
    "slice merge weights e^(M - m)": ("merge_slices", merge_slices_k(flip=True)),
    "output projection rows of the KV head": ("decode_out", decode_out_k(kv_rows=True)),
    "eq. 14 bit widths swapped": ("eq14_mean_bits", eq14_k(swap=True)),
    "eq. 16 drops the exempt layers": ("eq16_retained_fraction", eq16_k(drop_exempt=True)),
}


def _plant(monkeypatch, name, fn):
    monkeypatch.setattr(OM, name, fn)
    monkeypatch.setattr(O, name, fn)


@pytest.mark.parametrize("name", sorted(FAITHFUL))
def test_unplanted_copies_pass_their_pins(monkeypatch, name):
    _plant(monkeypatch, name, FAITHFUL[name])
    for pin in PINS[name]:
        pin()


@pytest.mark.parametrize("case", list(PLANTS))
def test_planted_mistake_fails_a_pin(monkeypatch, case):
    name, fn = PLANTS[case]
    _plant(monkeypatch, name, fn)
    caught = 0
    for pin in PINS[name]:
        try:
            with np.errstate(all="ignore"):
                pin()
        except AssertionError:
            caught += 1
    assert caught, f"no pin of {name} caught: {case}"
