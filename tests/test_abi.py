"""C ABI checks that need no GPU: the library loads, exports every function the
header declares, and its host-only logic (config checks, cache layout) agrees
with the oracle's byte accounting."""
import ctypes
import os
import re

import pytest

import oracle as O
from harness import gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "starkv.h")


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^STARKV_API[^;(]*?\b(starkv_\w+)\s*\(", txt, flags=re.M)))


@pytest.fixture(scope="module")
def S():
    from rank_mixed_precision_b200 import starkv
    starkv.lib()
    return starkv


def test_every_declared_symbol_is_exported(S):
    names = _declared()
    assert len(names) >= 13
    lib = ctypes.CDLL(S.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(S.EXPORTS) == names


def test_version(S):
    assert "sm_100a" in S.starkv_version()


def _cfg(S, w, max_position=1024):
    return S.make_config(w.H, w.h_kv, w.d_h, w.hidden, w.r_k, w.R, max_position, w.top_fraction, w.rope_base)


@pytest.mark.parametrize("i", range(5))
def test_cache_layout_matches_oracle(S, i):
    w = gen.workload(i)
    got = S.starkv_cache_layout(_cfg(S, w), 7)
    want = O.layout_sizes(O.config_of(w), 7)
    for k in ("k_codes", "v_codes", "k_meta", "v_meta"):
        assert got[k + "_bytes"] == want[k]
    cfg = O.config_of(w)
    assert got["key_group_size"] == cfg.key.g and got["value_group_size"] == cfg.val.g
    assert got["key_top"] == cfg.key.n_top and got["value_top"] == cfg.val.n_top
    assert got["key_region_bytes"] == cfg.key.region_bytes
    assert got["value_region_bytes"] == cfg.val.region_bytes


def test_top_fraction_0_2_rejected_for_supported_key_ranks(S):
    # a 20:80 split of r_k in {16, 32, 48, 64} leaves n_top in {3, 6, 10, 13}: group size < 4
    for rk in (16, 32, 48, 64):
        assert O.latent_split(rk, 0.2).g < 4
        with pytest.raises(S.StarKVError) as e:
            S.starkv_cache_layout(S.make_config(4, 4, 128, 256, rk, 80, 64, 0.2, 1e4), 1)
        assert e.value.code == 2


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 96, 2), ("num_kv_heads", 3, 2), ("rank_k", 24, 2), ("rank_v", 0, 1),
    ("hidden", 100, 2), ("flags", 2, 1), ("rope_base", 1.0, 1), ("top_fraction", 1.5, 1),
    ("max_position", 0, 1), ("max_position", (1 << 24) + 1, 2),
    ("num_kv_heads", 1 << 30, 2), ("num_q_heads", 2048, 2), ("hidden", 1 << 17, 2),
])
def test_config_rejections(S, field, value, code):
    c = _cfg(S, gen.workload(1))
    setattr(c, field, value)
    with pytest.raises(S.StarKVError) as e:
        S.starkv_cache_layout(c, 1)
    assert e.value.code == code
    assert S.starkv_last_error()


def test_group_size_must_be_supported(S):
    # r_k = 48: n_top = 12, n_bot = 36 -> g = 4 (allowed); R = 16 * 7 = 112: n_top = 28 -> g = 4
    assert S.starkv_cache_layout(S.make_config(4, 4, 64, 256, 48, 112, 64), 1)["key_group_size"] == 4
    # top_fraction 0.1 of 32 -> n_top 3 -> g = 1: rejected
    with pytest.raises(S.StarKVError):
        S.starkv_cache_layout(S.make_config(4, 4, 64, 256, 32, 64, 64, 0.1), 1)


def test_missing_library_fails_loudly(monkeypatch):
    from rank_mixed_precision_b200 import starkv
    monkeypatch.setattr(starkv, "_lib", None)
    monkeypatch.setattr(starkv, "LIB_PATH", "/nonexistent/libstarkv.so")
    with pytest.raises(ImportError):
        starkv.starkv_version()


def test_selftest_wait_timeout_checks_arguments_on_the_host(S):
    # raw call (no stream lookup): the context and the limit are checked before any launch
    assert S.lib().starkv_selftest_wait_timeout(None, 1_000_000, None) == S.ERR_INVALID_ARG


def test_every_entry_point_rejects_a_null_context_before_any_device_work(S):
    """Raw C calls with NULL handles: each returns INVALID_ARG (and sets a message)
    from the host-side checks, without a device or a CUDA call."""
    L = S.lib()
    sz = ctypes.c_size_t()
    u32 = ctypes.c_uint32()
    calls = {
        "starkv_append": lambda: L.starkv_append(None, None, None, None, 0, None, None),
        "starkv_decode_attn": lambda: L.starkv_decode_attn(None, None, None, None, None, 1, 1, None, None, 0, None),
        "starkv_decode_attn_noalloc": lambda: L.starkv_decode_attn_noalloc(None, None, None, None, None, 1, 1, None, None),
        "starkv_decode_attn_slice": lambda: L.starkv_decode_attn_slice(None, None, None, None, None, None, None, 1, 1,
                                                                      None, None, None, 0, None),
        "starkv_merge_slices": lambda: L.starkv_merge_slices(None, None, None, 1, 1, None, None),
        "starkv_set_output_projection": lambda: L.starkv_set_output_projection(None, None, 64, None),
        "starkv_decode_attn_out": lambda: L.starkv_decode_attn_out(None, None, None, None, None, 1, 1, None, None, 0,
                                                                  None),
        "starkv_prefill_attn": lambda: L.starkv_prefill_attn(None, None, None, None, None, None, 1, 1, 1, 1, None, None,
                                                            0, None),
        "starkv_workspace_bytes": lambda: L.starkv_workspace_bytes(None, 0, 1, 1, 0, ctypes.byref(sz)),
        "starkv_quantize_pack": lambda: L.starkv_quantize_pack(None, 0, None, 0, None, None, None),
        "starkv_dequantize": lambda: L.starkv_dequantize(None, 0, None, None, 0, None, None),
        "starkv_read_device_status": lambda: L.starkv_read_device_status(None, None, ctypes.byref(u32)),
        "starkv_get_config": lambda: L.starkv_get_config(None, None),
        "starkv_cache_layout": lambda: L.starkv_cache_layout(None, 1, None),
        "starkv_create": lambda: L.starkv_create(None, None, None, None, None, None, None),
        "starkv_selftest_wait_timeout": lambda: L.starkv_selftest_wait_timeout(None, 1_000_000, None),
    }
    assert set(calls) | {"starkv_version", "starkv_last_error", "starkv_destroy"} == set(S.EXPORTS)
    for name, call in calls.items():
        assert call() == S.ERR_INVALID_ARG, name
        assert S.starkv_last_error(), name
    assert L.starkv_destroy(None) == S.OK  # destroying nothing is allowed
