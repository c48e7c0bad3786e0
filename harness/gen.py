"""Seeded synthetic inputs for the STAR-KV latent-cache attention path.

This module only draws random numbers and rounds them to the storage types the
library accepts (bf16 for hidden states, queries and factors).  It holds none
of the method's arithmetic: no projection, rotation, quantisation, packing,
RoPE or attention.  Both the fp64 oracle (via the tests) and the CUDA library
(via the tests and the benchmark) consume what it produces.

Recipe (one PCG64 child stream per tensor, spawned from one seed):

* hidden states X ~ N(0, 1);
* down-projections A ~ N(0, 1/hidden); inside every latent (each KV head's
  key latent, and the joint value latent) column j is scaled by (j+1)^-1/2
  and two RNG-chosen outlier columns are scaled by 8, mimicking the
  singular-value ordering of an SVD-derived factor (STAR-KV technical review,
  section 2.2, eq. 2) with a few outlier channels (section 6.1);
* up-projections B_k,h = Q^T from the QR factorisation of a d_h x r_k
  Gaussian, B_v = Q^T from the QR of an (h_kv d_h) x R Gaussian, so their rows
  are orthonormal before the bf16 rounding;
* queries q ~ N(0, 1);
* latents drawn directly (for filling a cache without running the
  projection): N(0, 1) with the same per-column scale and outliers, which is
  the distribution X A has under the recipe above;
* paged cache: each sequence's pages are a random subset of a shuffled page
  pool, as a paged KV-cache allocator would hand them out.
"""
from __future__ import annotations

import dataclasses
import numpy as np

PAGE_TOKENS = 16

# Stable spawn indices: adding a tensor never changes the others' streams.
_STREAM = {
    "A_k": 1, "A_v": 2, "B_k": 3, "B_v": 4, "X": 5, "q": 6, "latent_k": 7,
    "latent_v": 8, "pages": 9, "lens": 10, "outlier_k": 11, "outlier_v": 12,
    "X_chunk": 13, "q_chunk": 14, "X_step": 15, "q_step": 16,
}


def rng_for(name: str, seed: int = 0, sub: int = 0) -> np.random.Generator:
    """Independent PCG64 stream for tensor ``name`` (and sub-index ``sub``)."""
    ss = np.random.SeedSequence(entropy=seed, spawn_key=(_STREAM[name], sub))
    return np.random.Generator(np.random.PCG64(ss))


# ----------------------------------------------------------------------------
# bf16 storage rounding (round to nearest even), as the library stores inputs.
# ----------------------------------------------------------------------------
def bf16_bits(x) -> np.ndarray:
    """Round float32 values to bf16, returning the raw uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    """float32 value of bf16 bit patterns (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def to_bf16(x) -> tuple[np.ndarray, np.ndarray]:
    """(float32 values representable in bf16, their uint16 bit patterns)."""
    b = bf16_bits(x)
    return bf16_value(b), b


# ----------------------------------------------------------------------------
# Workload descriptions (shapes only; no weights or datasets are involved).
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    H: int            # query heads
    h_kv: int         # KV heads
    d_h: int          # head dim
    hidden: int       # model width of X
    r_k: int          # key latent rank per KV head
    R: int            # joint value latent rank
    batch: int
    ctx: int          # context length (upper bound when ragged)
    ctx_lo: int = 0   # >0: lengths ~ U[ctx_lo, ctx]
    rope_base: float = 10000.0
    top_fraction: float = 0.25
    steps: int = 0    # decode steps with one appended token each (long-context run)
    chunk: int = 0    # prefill: tokens appended then attended causally
    fp16_latent: bool = False  # the unquantised storage variant
    key_ranks: tuple = None    # ragged key ranks, one per KV head (r_k = their maximum)


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_h4_d64_r16_R64_b1_t256", H=4, h_kv=4, d_h=64, hidden=256,
                 r_k=16, R=64, batch=1, ctx=256),
        Workload("longchat7b_decode_b16_t4096", H=32, h_kv=32, d_h=128, hidden=4096,
                 r_k=32, R=1024, batch=16, ctx=4096),
        Workload("longchat7b_stream_b1_t32768_s128", H=32, h_kv=32, d_h=128,
                 hidden=4096, r_k=32, R=1024, batch=1, ctx=32768, steps=128),
        Workload("llama3_8b_gqa_decode_b32_t4096to8192", H=32, h_kv=8, d_h=128,
                 hidden=4096, r_k=64, R=512, batch=32, ctx=8192, ctx_lo=4096,
                 rope_base=500000.0),
        Workload("longchat7b_prefill_b4_t30720_c2048", H=32, h_kv=32, d_h=128,
                 hidden=4096, r_k=32, R=1024, batch=4, ctx=30720, chunk=2048),
    ]
}
WORKLOAD_ORDER = list(WORKLOADS)


def workload(i_or_name) -> Workload:
    if isinstance(i_or_name, int):
        return WORKLOADS[WORKLOAD_ORDER[i_or_name]]
    return WORKLOADS[i_or_name]


def shrink(w: Workload, **kw) -> Workload:
    return dataclasses.replace(w, **kw)


# ----------------------------------------------------------------------------
# Tensors
# ----------------------------------------------------------------------------
def _latent_scale(r: int, rng: np.random.Generator) -> tuple[np.ndarray, np.ndarray]:
    """Per-column scale (j+1)^-1/2 with two outlier columns x8."""
    scale = 1.0 / np.sqrt(np.arange(1, r + 1, dtype=np.float64))
    out = rng.choice(r, size=min(2, r), replace=False)
    scale[out] *= 8.0
    return scale, np.sort(out)


@dataclasses.dataclass
class Factors:
    A_k: np.ndarray   # [hidden, h_kv*r_k] float32 (bf16 values)
    A_v: np.ndarray   # [hidden, R]
    B_k: np.ndarray   # [h_kv, r_k, d_h]
    B_v: np.ndarray   # [R, h_kv*d_h]
    outliers_k: list  # per KV head, the two outlier columns
    outliers_v: list

    def bits(self):
        return {k: bf16_bits(getattr(self, k)) for k in ("A_k", "A_v", "B_k", "B_v")}


def key_ranks_of(w: Workload):
    return list(w.key_ranks) if w.key_ranks is not None else [w.r_k] * w.h_kv


def make_factors(w: Workload, seed: int = 0, a_std: float | None = None) -> Factors:
    """Factors in the library's layout.  With ragged key ranks, A_k holds
    sum_h r_h columns and B_k is [sum_h r_h, d_h] (head h's rows after the
    earlier heads'); with uniform ranks B_k is [h_kv, r_k, d_h]."""
    hidden = w.hidden
    std = (1.0 / np.sqrt(hidden)) if a_std is None else a_std
    if w.key_ranks is not None:
        return _make_factors_ragged(w, seed, std)
    rk = rng_for("A_k", seed)
    ok = rng_for("outlier_k", seed)
    A_k = np.empty((hidden, w.h_kv * w.r_k), np.float64)
    outk = []
    for h in range(w.h_kv):
        sc, o = _latent_scale(w.r_k, ok)
        A_k[:, h * w.r_k:(h + 1) * w.r_k] = rk.standard_normal((hidden, w.r_k)) * std * sc
        outk.append(o.tolist())
    rv = rng_for("A_v", seed)
    sc, outv = _latent_scale(w.R, rng_for("outlier_v", seed))
    A_v = rv.standard_normal((hidden, w.R)) * std * sc
    rb = rng_for("B_k", seed)
    B_k = np.empty((w.h_kv, w.r_k, w.d_h), np.float64)
    for h in range(w.h_kv):
        Q, _ = np.linalg.qr(rb.standard_normal((w.d_h, w.r_k)))
        B_k[h] = Q.T
    Q, _ = np.linalg.qr(rng_for("B_v", seed).standard_normal((w.h_kv * w.d_h, w.R)))
    B_v = Q.T
    f = lambda a: to_bf16(a.astype(np.float32))[0]
    return Factors(f(A_k), f(A_v), f(B_k), f(B_v), outk, outv.tolist())


def _make_factors_ragged(w: Workload, seed: int, std: float) -> Factors:
    ranks = key_ranks_of(w)
    hidden = w.hidden
    rk, ok, rb = rng_for("A_k", seed), rng_for("outlier_k", seed), rng_for("B_k", seed)
    A_k = np.empty((hidden, sum(ranks)), np.float64)
    B_k = np.empty((sum(ranks), w.d_h), np.float64)
    outk, col = [], 0
    for r in ranks:
        sc, o = _latent_scale(r, ok)
        A_k[:, col:col + r] = rk.standard_normal((hidden, r)) * std * sc
        Q, _ = np.linalg.qr(rb.standard_normal((w.d_h, r)))
        B_k[col:col + r] = Q.T
        outk.append(o.tolist())
        col += r
    rv = rng_for("A_v", seed)
    sc, outv = _latent_scale(w.R, rng_for("outlier_v", seed))
    A_v = rv.standard_normal((hidden, w.R)) * std * sc
    Q, _ = np.linalg.qr(rng_for("B_v", seed).standard_normal((w.h_kv * w.d_h, w.R)))
    f = lambda a: to_bf16(a.astype(np.float32))[0]
    return Factors(f(A_k), f(A_v), f(B_k), f(Q.T), outk, outv.tolist())


def make_hidden(n: int, hidden: int, seed: int = 0, name: str = "X", sub: int = 0):
    """Hidden states X ~ N(0,1), bf16 values as float32 [n, hidden]."""
    x = rng_for(name, seed, sub).standard_normal((n, hidden), dtype=np.float32)
    return to_bf16(x)[0]


def make_queries(n: int, H: int, d_h: int, seed: int = 0, name: str = "q", sub: int = 0):
    """Queries q ~ N(0,1) (pre-RoPE), bf16 values as float32 [n, H, d_h]."""
    q = rng_for(name, seed, sub).standard_normal((n, H, d_h), dtype=np.float32)
    return to_bf16(q)[0]


def make_latents(w: Workload, n: int, seed: int = 0, sub: int = 0):
    """Pre-rotation latents (float32) for n tokens, as X A would produce them.

    Returns (z_k [n, h_kv, r_k], z_v [n, R]).
    """
    ok = rng_for("outlier_k", seed)
    if w.key_ranks is not None:
        # ragged ranks: head h's first r_h channels, zero past its rank
        sk = np.zeros((w.h_kv, w.r_k))
        for h, r in enumerate(key_ranks_of(w)):
            sk[h, :r] = _latent_scale(r, ok)[0]
    else:
        sk = np.stack([_latent_scale(w.r_k, ok)[0] for _ in range(w.h_kv)])
    sv = _latent_scale(w.R, rng_for("outlier_v", seed))[0]
    zk = rng_for("latent_k", seed, sub).standard_normal((n, w.h_kv, w.r_k)) * sk
    zv = rng_for("latent_v", seed, sub).standard_normal((n, w.R)) * sv
    return zk.astype(np.float32), zv.astype(np.float32)


def make_seq_lens(w: Workload, seed: int = 0) -> np.ndarray:
    if w.ctx_lo > 0:
        return rng_for("lens", seed).integers(w.ctx_lo, w.ctx + 1, size=w.batch).astype(np.int32)
    return np.full(w.batch, w.ctx, np.int32)


def make_block_table(seq_caps, seed: int = 0, extra_pages: int = 0):
    """Random page assignment.

    seq_caps: per sequence, the number of tokens its pages must hold.
    Returns (block_table [B, max_pages] int32 with -1 padding, n_pages).
    """
    need = [(int(c) + PAGE_TOKENS - 1) // PAGE_TOKENS for c in seq_caps]
    total = sum(need) + extra_pages
    perm = rng_for("pages", seed).permutation(total).astype(np.int32)
    max_pages = max(need) if need else 0
    bt = np.full((len(need), max(max_pages, 1)), -1, np.int32)
    off = 0
    for b, k in enumerate(need):
        bt[b, :k] = perm[off:off + k]
        off += k
    return bt, total


def slots_for(block_table: np.ndarray, b: int, positions) -> np.ndarray:
    """Physical slot (page*16 + offset) of token positions of sequence b."""
    positions = np.asarray(positions, np.int64)
    return block_table[b, positions // PAGE_TOKENS].astype(np.int64) * PAGE_TOKENS + positions % PAGE_TOKENS
