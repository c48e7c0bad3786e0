"""Python binding of the STAR-KV C ABI (include/starkv.h).

Argument marshalling only: every step of the computation runs in the CUDA
library ``libstarkv.so``.  Functions carry the C names and take torch tensors
(device memory and streams come from PyTorch).  If the library is missing the
import of this module still succeeds, but every call raises: there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libstarkv.so")

PAGE_TOKENS = 16
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_WORKSPACE_TOO_SMALL, ERR_CUDA, ERR_DEVICE_STATUS = range(6)
DEV_BAD_PAGE, DEV_BAD_SEQ_LEN, DEV_QUANT_OVERFLOW, DEV_BAD_SLOT, DEV_BAD_QUERY_SPAN, DEV_WAIT_TIMEOUT = 1, 2, 4, 8, 16, 32
OP_DECODE, OP_PREFILL, OP_DECODE_OUT = 0, 1, 2
LATENT_KEY, LATENT_VALUE = 0, 1

# every function include/starkv.h declares
EXPORTS = [
    "starkv_version", "starkv_last_error", "starkv_cache_layout", "starkv_create", "starkv_destroy",
    "starkv_get_config", "starkv_append", "starkv_workspace_bytes", "starkv_decode_attn",
    "starkv_decode_attn_noalloc", "starkv_decode_attn_slice", "starkv_merge_slices",
    "starkv_set_output_projection", "starkv_decode_attn_out",
    "starkv_prefill_attn", "starkv_quantize_pack", "starkv_dequantize", "starkv_read_device_status",
    "starkv_selftest_wait_timeout",
]


class starkv_config(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("rank_k", ctypes.c_int32), ("rank_v", ctypes.c_int32),
                ("max_position", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("top_fraction", ctypes.c_double), ("rope_base", ctypes.c_double),
                ("key_ranks", ctypes.POINTER(ctypes.c_int32))]


class starkv_cache(ctypes.Structure):
    _fields_ = [("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("k_meta", ctypes.c_void_p), ("v_meta", ctypes.c_void_p),
                ("n_pages", ctypes.c_int64)]


class starkv_cache_sizes(ctypes.Structure):
    _fields_ = [("k_codes_bytes", ctypes.c_int64), ("v_codes_bytes", ctypes.c_int64),
                ("k_meta_bytes", ctypes.c_int64), ("v_meta_bytes", ctypes.c_int64),
                ("key_region_bytes", ctypes.c_int32), ("value_region_bytes", ctypes.c_int32),
                ("key_group_size", ctypes.c_int32), ("value_group_size", ctypes.c_int32),
                ("key_top", ctypes.c_int32), ("value_top", ctypes.c_int32),
                ("key_groups", ctypes.c_int32), ("value_groups", ctypes.c_int32),
                ("key_page_bytes", ctypes.c_int32), ("key_page_meta_bytes", ctypes.c_int32)]


class StarKVError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"starkv error {code}: {msg}")
        self.code = code


_lib = None
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_SIGS = {
    "starkv_version": ([], ctypes.c_char_p),
    "starkv_last_error": ([], ctypes.c_char_p),
    "starkv_cache_layout": ([ctypes.POINTER(starkv_config), _i64, ctypes.POINTER(starkv_cache_sizes)], _i32),
    "starkv_create": ([ctypes.POINTER(starkv_config), _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(_vp)], _i32),
    "starkv_destroy": ([_vp], _i32),
    "starkv_get_config": ([_vp, ctypes.POINTER(starkv_config)], _i32),
    "starkv_append": ([_vp, ctypes.POINTER(starkv_cache), _vp, _vp, _i64, _vp, _vp], _i32),
    "starkv_workspace_bytes": ([_vp, _i32, _i32, _i32, _i64, ctypes.POINTER(_sz)], _i32),
    "starkv_decode_attn": ([_vp, ctypes.POINTER(starkv_cache), _vp, _vp, _vp, _i32, _i32, _vp, _vp, _sz, _vp], _i32),
    "starkv_decode_attn_noalloc": ([_vp, ctypes.POINTER(starkv_cache), _vp, _vp, _vp, _i32, _i32, _vp, _vp], _i32),
    "starkv_decode_attn_slice": ([_vp, ctypes.POINTER(starkv_cache), _vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp,
                                  _vp, _sz, _vp], _i32),
    "starkv_merge_slices": ([_vp, _vp, _vp, _i32, _i32, _vp, _vp], _i32),
    "starkv_set_output_projection": ([_vp, _vp, _i32, _vp], _i32),
    "starkv_decode_attn_out": ([_vp, ctypes.POINTER(starkv_cache), _vp, _vp, _vp, _i32, _i32, _vp, _vp, _sz, _vp],
                               _i32),
    "starkv_prefill_attn": ([_vp, ctypes.POINTER(starkv_cache), _vp, _vp, _vp, _vp, _i32, _i32, _i64, _i32, _vp,
                             _vp, _sz, _vp], _i32),
    "starkv_quantize_pack": ([_vp, _i32, _vp, _i64, _vp, _vp, _vp], _i32),
    "starkv_dequantize": ([_vp, _i32, _vp, _vp, _i64, _vp, _vp], _i32),
    "starkv_read_device_status": ([_vp, _vp, ctypes.POINTER(ctypes.c_uint32)], _i32),
    "starkv_selftest_wait_timeout": ([_vp, ctypes.c_uint64, _vp], _i32),
}


def lib() -> ctypes.CDLL:
    """Load libstarkv.so (raises when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m rank_mixed_precision_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(st: int):
    if st != OK:
        raise StarKVError(st, lib().starkv_last_error().decode())


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


# ---------------------------------------------------------------------------
FLAG_FP16_LATENT = 1


def make_config(H, h_kv, d_h, hidden, r_k, R, max_position, top_fraction=0.25, rope_base=10000.0, flags=0,
                key_ranks=None):
    """key_ranks: optional per-KV-head key ranks (ragged ranks; r_k must be their maximum)."""
    cfg = starkv_config(H, h_kv, d_h, hidden, r_k, R, max_position, flags, top_fraction, rope_base, None)
    if key_ranks is not None:
        arr = (ctypes.c_int32 * len(key_ranks))(*[int(r) for r in key_ranks])
        cfg.key_ranks = ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32))
        cfg._key_ranks_keepalive = arr
    return cfg


def LATENT_KEY_HEAD(h: int) -> int:
    """Latent kind of KV head h's key latent for starkv_quantize_pack / starkv_dequantize."""
    return 2 + h


def starkv_version() -> str:
    return lib().starkv_version().decode()


def starkv_last_error() -> str:
    return lib().starkv_last_error().decode()


def starkv_cache_layout(cfg: starkv_config, n_pages: int) -> dict:
    out = starkv_cache_sizes()
    _check(lib().starkv_cache_layout(ctypes.byref(cfg), n_pages, ctypes.byref(out)))
    return {f: getattr(out, f) for f, _ in starkv_cache_sizes._fields_}


def starkv_create(cfg: starkv_config, A_k, A_v, B_k, B_v, stream=None):
    for t, n in ((A_k, "A_k"), (A_v, "A_v"), (B_k, "B_k"), (B_v, "B_v")):
        _need(t, torch.bfloat16, n)
    if cfg.key_ranks:
        kcols = sum(cfg.key_ranks[h] for h in range(cfg.num_kv_heads))
        want_bk = (kcols, cfg.head_dim)          # ragged ranks: head h's rows after the earlier heads'
    else:
        kcols = cfg.num_kv_heads * cfg.rank_k
        want_bk = (cfg.num_kv_heads, cfg.rank_k, cfg.head_dim)
    if tuple(A_k.shape) != (cfg.hidden, kcols):
        raise ValueError(f"A_k shape {tuple(A_k.shape)}")
    if tuple(A_v.shape) != (cfg.hidden, cfg.rank_v):
        raise ValueError(f"A_v shape {tuple(A_v.shape)}")
    if tuple(B_k.shape) != want_bk:
        raise ValueError(f"B_k shape {tuple(B_k.shape)}")
    if tuple(B_v.shape) != (cfg.rank_v, cfg.num_kv_heads * cfg.head_dim):
        raise ValueError(f"B_v shape {tuple(B_v.shape)}")
    h = ctypes.c_void_p()
    _check(lib().starkv_create(ctypes.byref(cfg), _p(A_k), _p(A_v), _p(B_k), _p(B_v), _stream(stream),
                               ctypes.byref(h)))
    return h


def starkv_destroy(ctx):
    _check(lib().starkv_destroy(ctx))


def starkv_get_config(ctx) -> starkv_config:
    out = starkv_config()
    _check(lib().starkv_get_config(ctx, ctypes.byref(out)))
    return out


def starkv_append(ctx, cache: starkv_cache, X, slot_mapping, latents_out=None, stream=None):
    _need(X, torch.bfloat16, "X", 2)
    _need(slot_mapping, torch.int64, "slot_mapping", 1)
    if slot_mapping.shape[0] != X.shape[0]:
        raise ValueError("slot_mapping and X disagree on n")
    if latents_out is not None:
        _need(latents_out, torch.float32, "latents_out", 2)
    _check(lib().starkv_append(ctx, ctypes.byref(cache), _p(X), _p(slot_mapping), X.shape[0], _p(latents_out),
                               _stream(stream)))


def starkv_workspace_bytes(ctx, op: int, batch: int, max_pages: int, total_q: int = 0) -> int:
    out = ctypes.c_size_t()
    _check(lib().starkv_workspace_bytes(ctx, op, batch, max_pages, total_q, ctypes.byref(out)))
    return out.value


def starkv_decode_attn(ctx, cache: starkv_cache, q, block_table, seq_lens, out, workspace, stream=None):
    _need(q, torch.bfloat16, "q", 3)
    _need(block_table, torch.int32, "block_table", 2)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    _need(out, torch.bfloat16, "out", 3)
    _need(workspace, torch.uint8, "workspace", 1)
    B = q.shape[0]
    if block_table.shape[0] != B or seq_lens.shape[0] != B or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q / block_table / seq_lens / out disagree on the batch")
    _check(lib().starkv_decode_attn(ctx, ctypes.byref(cache), _p(q), _p(block_table), _p(seq_lens), B,
                                    block_table.shape[1], _p(out), _p(workspace), workspace.numel(),
                                    _stream(stream)))


def starkv_decode_attn_noalloc(ctx, cache: starkv_cache, q, block_table, seq_lens, out, stream=None):
    """Decode with the library's built-in scratch instead of a caller workspace
    (for callers that cannot allocate device memory; see include/starkv.h)."""
    _need(q, torch.bfloat16, "q", 3)
    _need(block_table, torch.int32, "block_table", 2)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    _need(out, torch.bfloat16, "out", 3)
    B = q.shape[0]
    if block_table.shape[0] != B or seq_lens.shape[0] != B or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q / block_table / seq_lens / out disagree on the batch")
    _check(lib().starkv_decode_attn_noalloc(ctx, ctypes.byref(cache), _p(q), _p(block_table), _p(seq_lens), B,
                                            block_table.shape[1], _p(out), _stream(stream)))


def starkv_decode_attn_slice(ctx, cache: starkv_cache, q, block_table, seq_lens, key_pos0, q_pos, out_o, out_ml,
                             workspace, stream=None):
    """Decode over one slice of each sequence's context (sequence sharding):
    fp32 output normalised within the slice and its (m, l) statistics."""
    _need(q, torch.bfloat16, "q", 3)
    _need(block_table, torch.int32, "block_table", 2)
    for t, n in ((seq_lens, "seq_lens"), (key_pos0, "key_pos0"), (q_pos, "q_pos")):
        _need(t, torch.int32, n, 1)
    _need(out_o, torch.float32, "out_o", 3)
    _need(out_ml, torch.float32, "out_ml", 3)
    _need(workspace, torch.uint8, "workspace", 1)
    B = q.shape[0]
    if any(t.shape[0] != B for t in (block_table, seq_lens, key_pos0, q_pos, out_ml)) or \
            tuple(out_o.shape) != tuple(q.shape) or tuple(out_ml.shape) != (B, q.shape[1], 2):
        raise ValueError("slice decode arguments disagree on the shapes")
    _check(lib().starkv_decode_attn_slice(ctx, ctypes.byref(cache), _p(q), _p(block_table), _p(seq_lens),
                                          _p(key_pos0), _p(q_pos), B, block_table.shape[1], _p(out_o), _p(out_ml),
                                          _p(workspace), workspace.numel(), _stream(stream)))


def starkv_set_output_projection(ctx, W_o, stream=None):
    """W_o: bf16 [num_q_heads * head_dim, model_dim] (copied by the library)."""
    _need(W_o, torch.bfloat16, "W_o", 2)
    _check(lib().starkv_set_output_projection(ctx, _p(W_o), W_o.shape[1], _stream(stream)))


def starkv_decode_attn_out(ctx, cache: starkv_cache, q, block_table, seq_lens, y, workspace, stream=None):
    """Decode attention and the output projection: y bf16 [batch, model_dim]."""
    _need(q, torch.bfloat16, "q", 3)
    _need(block_table, torch.int32, "block_table", 2)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    _need(y, torch.bfloat16, "y", 2)
    _need(workspace, torch.uint8, "workspace", 1)
    B = q.shape[0]
    if block_table.shape[0] != B or seq_lens.shape[0] != B or y.shape[0] != B:
        raise ValueError("q / block_table / seq_lens / y disagree on the batch")
    _check(lib().starkv_decode_attn_out(ctx, ctypes.byref(cache), _p(q), _p(block_table), _p(seq_lens), B,
                                        block_table.shape[1], _p(y), _p(workspace), workspace.numel(),
                                        _stream(stream)))


def starkv_merge_slices(ctx, o_parts, ml_parts, out, stream=None):
    """Merge slice results [n, B, H, d] / [n, B, H, 2] into the bf16 output [B, H, d]."""
    _need(o_parts, torch.float32, "o_parts", 4)
    _need(ml_parts, torch.float32, "ml_parts", 4)
    _need(out, torch.bfloat16, "out", 3)
    n, B = o_parts.shape[0], o_parts.shape[1]
    if tuple(o_parts.shape[1:]) != tuple(out.shape) or tuple(ml_parts.shape) != (n, B, out.shape[1], 2):
        raise ValueError("merge arguments disagree on the shapes")
    _check(lib().starkv_merge_slices(ctx, _p(o_parts), _p(ml_parts), n, B, _p(out), _stream(stream)))


def starkv_prefill_attn(ctx, cache: starkv_cache, q, cu_q, block_table, seq_lens, max_q_len, out, workspace,
                        stream=None):
    _need(q, torch.bfloat16, "q", 3)
    _need(cu_q, torch.int32, "cu_q", 1)
    _need(block_table, torch.int32, "block_table", 2)
    _need(seq_lens, torch.int32, "seq_lens", 1)
    _need(out, torch.bfloat16, "out", 3)
    _need(workspace, torch.uint8, "workspace", 1)
    B = seq_lens.shape[0]
    if cu_q.shape[0] != B + 1 or block_table.shape[0] != B:
        raise ValueError("cu_q / block_table / seq_lens disagree on the batch")
    _check(lib().starkv_prefill_attn(ctx, ctypes.byref(cache), _p(q), _p(cu_q), _p(block_table), _p(seq_lens), B,
                                     block_table.shape[1], q.shape[0], max_q_len, _p(out), _p(workspace),
                                     workspace.numel(), _stream(stream)))


def starkv_quantize_pack(ctx, which: int, z, codes, meta, stream=None):
    _need(z, torch.float32, "z", 2)
    _need(codes, torch.uint8, "codes")
    _need(meta, torch.int32, "meta")
    _check(lib().starkv_quantize_pack(ctx, which, _p(z), z.shape[0], _p(codes), _p(meta), _stream(stream)))


def starkv_dequantize(ctx, which: int, codes, meta, n: int, z_out, stream=None):
    _need(codes, torch.uint8, "codes")
    _need(meta, torch.int32, "meta")
    _need(z_out, torch.float32, "z_out", 2)
    _check(lib().starkv_dequantize(ctx, which, _p(codes), _p(meta), n, _p(z_out), _stream(stream)))


def starkv_selftest_wait_timeout(ctx, limit_ns: int, stream=None) -> None:
    _check(lib().starkv_selftest_wait_timeout(ctx, int(limit_ns), _stream(stream)))


def starkv_read_device_status(ctx, stream=None) -> int:
    """Status word (0 = clean).  Does not raise on a non-zero word."""
    v = ctypes.c_uint32()
    st = lib().starkv_read_device_status(ctx, _stream(stream), ctypes.byref(v))
    if st not in (OK, ERR_DEVICE_STATUS):
        _check(st)
    return v.value


# ---------------------------------------------------------------------------
# Convenience wrappers (allocation through torch; no arithmetic)
# ---------------------------------------------------------------------------
class LatentCache:
    """The four page pools of a paged latent cache, allocated with torch."""

    def __init__(self, cfg: starkv_config, n_pages: int, device="cuda"):
        self.sizes = starkv_cache_layout(cfg, n_pages)
        self.n_pages = n_pages
        mk = lambda nbytes: torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=device)
        self.k_codes = mk(self.sizes["k_codes_bytes"])
        self.v_codes = mk(self.sizes["v_codes_bytes"])
        self.k_meta = mk(self.sizes["k_meta_bytes"])
        self.v_meta = mk(self.sizes["v_meta_bytes"])
        self.struct = starkv_cache(self.k_codes.data_ptr(), self.v_codes.data_ptr(), self.k_meta.data_ptr(),
                                   self.v_meta.data_ptr(), n_pages)

    def nbytes(self) -> int:
        return sum(self.sizes[k] for k in ("k_codes_bytes", "v_codes_bytes", "k_meta_bytes", "v_meta_bytes"))


class StarKV:
    """A context (prepared factors) plus workspace management."""

    def __init__(self, cfg: starkv_config, A_k, A_v, B_k, B_v, stream=None):
        self.cfg = cfg
        self.ctx = starkv_create(cfg, A_k, A_v, B_k, B_v, stream)
        self._ws = None

    def close(self):
        if self.ctx is not None:
            starkv_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace(self, op, batch, max_pages, total_q=0):
        n = starkv_workspace_bytes(self.ctx, op, batch, max_pages, total_q)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")
        return self._ws

    def new_cache(self, n_pages: int) -> LatentCache:
        return LatentCache(self.cfg, n_pages)

    def append(self, cache: LatentCache, X, slot_mapping, latents_out=None, stream=None):
        starkv_append(self.ctx, cache.struct, X, slot_mapping, latents_out, stream)

    def decode(self, cache: LatentCache, q, block_table, seq_lens, out=None, stream=None):
        out = torch.empty_like(q) if out is None else out
        ws = self.workspace(OP_DECODE, q.shape[0], block_table.shape[1])
        starkv_decode_attn(self.ctx, cache.struct, q, block_table, seq_lens, out, ws, stream)
        return out

    def prefill(self, cache: LatentCache, q, cu_q, block_table, seq_lens, max_q_len, out=None, stream=None):
        out = torch.empty_like(q) if out is None else out
        ws = self.workspace(OP_PREFILL, seq_lens.shape[0], block_table.shape[1], q.shape[0])
        starkv_prefill_attn(self.ctx, cache.struct, q, cu_q, block_table, seq_lens, max_q_len, out, ws, stream)
        return out

    def status(self, stream=None) -> int:
        return starkv_read_device_status(self.ctx, stream)
