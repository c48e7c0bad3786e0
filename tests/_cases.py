"""Shared builders for the GPU parity tests.

Inputs come from harness.gen (seeded); packed caches are written by the oracle
and uploaded byte for byte, so the CUDA path and the oracle read identical
caches.  Nothing here takes a value from the CUDA path into the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from harness import gen

# attention tolerance (fp32/fp16 arithmetic against the fp64 oracle):
# max-abs error <= 1e-2 and relative L2 error <= 5e-3
ATOL_MAX = 1e-2
REL_L2 = 5e-3


def bf16_tensor(a, device="cuda"):
    bits = gen.bf16_bits(np.asarray(a, np.float32))
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(device)


def skv():
    from rank_mixed_precision_b200 import starkv
    return starkv


def make_ctx(w: gen.Workload, seed=0, max_position=None):
    S = skv()
    f = gen.make_factors(w, seed)
    mp = max_position or (w.ctx + max(w.steps, w.chunk) + 16)
    cfg = S.make_config(w.H, w.h_kv, w.d_h, w.hidden, w.r_k, w.R, mp, w.top_fraction, w.rope_base,
                        S.FLAG_FP16_LATENT if w.fp16_latent else 0, w.key_ranks)
    kv = S.StarKV(cfg, bf16_tensor(f.A_k), bf16_tensor(f.A_v), bf16_tensor(f.B_k), bf16_tensor(f.B_v))
    return kv, f


def oracle_cache(w: gen.Workload, seq_lens, seed=0, extra_pages=0, caps=None):
    """Oracle-written cache holding positions [0, seq_lens[b]) of every sequence.

    caps: per-sequence token capacity of the page table (>= seq_lens).
    """
    cfg = O.config_of(w)
    caps = list(seq_lens) if caps is None else list(caps)
    bt, n_pages = gen.make_block_table(caps, seed, extra_pages)
    cache = O.new_cache(cfg, max(n_pages, 1))
    for b, L in enumerate(seq_lens):
        if L == 0:
            continue
        zk, zv = gen.make_latents(w, int(L), seed, sub=b)
        O.write_latents(cache, gen.slots_for(bt, b, np.arange(int(L))), zk, zv)
    return cfg, cache, bt, max(n_pages, 1)


def upload(lc, oc: O.Cache):
    """Copy an oracle cache's bytes into a LatentCache (same layout)."""
    for name in ("k_codes", "v_codes", "k_meta", "v_meta"):
        src = np.ascontiguousarray(getattr(oc, name)).view(np.uint8).reshape(-1)
        dst = getattr(lc, name)
        assert dst.numel() >= src.size
        dst[:src.size].copy_(torch.from_numpy(src))


def download(lc, oc_like: O.Cache) -> O.Cache:
    """Bytes of a LatentCache as an oracle-shaped cache (for byte comparisons)."""
    out = O.new_cache(oc_like.cfg, oc_like.k_codes.shape[0])
    for name in ("k_codes", "v_codes", "k_meta", "v_meta"):
        arr = getattr(out, name)
        raw = getattr(lc, name)[:arr.nbytes].cpu().numpy()
        arr[...] = raw.view(arr.dtype).reshape(arr.shape)
    return out


def check_attention(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    mask = ~np.isnan(ref)
    g, r = got[mask], ref[mask]
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - r)
    rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    assert err.max() <= ATOL_MAX, f"{what}: max-abs {err.max():.3e} > {ATOL_MAX}"
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e} > {REL_L2}"
    return float(err.max()), float(rel)
