"""The allocation-free decode entry point against the ordinary one.

starkv_decode_attn_noalloc serves callers that cannot call cudaMalloc (a plugin
inside a serving engine that owns all device memory, a loop that must never
enter the allocator): its split partials live in a built-in scratch array
instead of a caller workspace.  This file is named to be collected last so
that a run stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from harness import gen

import oracle as O
from _cases import ATOL_MAX, REL_L2, bf16_tensor, check_attention, make_ctx, oracle_cache, skv, upload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wi,lens", [(0, [256, 17, 1, 0]), (1, [300, 1000, 64]), (3, [700, 1500, 33])],
                         ids=["tiny", "longchat", "llama3gqa"])
def test_noalloc_matches_workspace_decode_twice(wi, lens):
    S = skv()
    w = gen.workload(wi)
    kv, f = make_ctx(w, max_position=max(lens) + 16)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, lens, extra_pages=2)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        q = bf16_tensor(gen.make_queries(len(lens), w.H, w.d_h))
        btd = torch.from_numpy(bt).cuda()
        sl = torch.tensor(np.asarray(lens, np.int32)).cuda()
        ref = kv.decode(lc, q, btd, sl).float()
        want = O.decode(oc, gen.make_queries(len(lens), w.H, w.d_h), f.B_k, f.B_v, bt, lens)
        for call in range(2):           # the scratch keeps the previous call's contents
            out = torch.full_like(q, float("nan"))
            S.starkv_decode_attn_noalloc(kv.ctx, lc.struct, q, btd, sl, out)
            got = out.float()
            assert torch.isfinite(got).all(), f"call {call}: non-finite output"
            err = (got - ref).abs().max().item()
            rel = (torch.linalg.norm(got - ref) / torch.linalg.norm(ref).clamp_min(1e-30)).item()
            assert err <= ATOL_MAX and rel <= REL_L2, f"call {call}: max-abs {err:.3e} rel-L2 {rel:.3e}"
            check_attention(got.cpu().numpy(), want, f"call {call} against the oracle")
        assert kv.status() == 0
    finally:
        kv.close()


def test_noalloc_rejects_shapes_beyond_its_scratch():
    S = skv()
    w = gen.workload(1)
    kv, f = make_ctx(w, max_position=64)
    try:
        lc = kv.new_cache(1)
        B = 4096                          # 4096 x 32 heads x (1024 + 2) x 4 B > 16 MiB of partials
        q = torch.zeros((B, w.H, w.d_h), dtype=torch.bfloat16, device="cuda")
        bt = torch.zeros((B, 1), dtype=torch.int32, device="cuda")
        sl = torch.ones(B, dtype=torch.int32, device="cuda")
        with pytest.raises(S.StarKVError) as e:
            S.starkv_decode_attn_noalloc(kv.ctx, lc.struct, q, bt, sl, torch.empty_like(q))
        assert e.value.code == S.ERR_UNSUPPORTED_SHAPE
        assert "scratch" in S.starkv_last_error()
    finally:
        kv.close()


SCRATCH = 16 << 20


def _simt_workspace(batch, H, R, max_pages):
    """Partials of the CUDA-core decode plan: batch * H * splits * (R + 2) * 4 bytes."""
    splits = min(-(-4 * 148 // (batch * H)), -(-max_pages // 16))
    splits = max(splits, 1)
    pps = max(-(-max_pages // splits), 1)
    return batch * H * (-(-max_pages // pps)) * (R + 2) * 4


def test_noalloc_at_the_largest_accepted_workspace():
    """A shape whose tensor-core workspace sits just under the 16 MiB scratch:
    the last bytes of the array are in use, so an offset past its end would show."""
    S = skv()
    w = gen.workload(0)                    # 4 heads, d_h 64, r_k 16, R 64: the tensor-core path
    B = 2
    kv0, _ = make_ctx(w, max_position=64)
    try:
        best = None
        for mp in range(1024, 40000, 256):
            ws = S.starkv_workspace_bytes(kv0.ctx, S.OP_DECODE, B, mp)
            if ws <= SCRATCH:
                best = (mp, ws)
            else:
                break
        assert best is not None
        mp, ws = best
        assert ws > SCRATCH - (1 << 20), f"largest accepted workspace {ws} is not near the scratch size"
        assert ws != _simt_workspace(B, w.H, w.R, mp)     # the tensor-core plan, not the CUDA-core one
    finally:
        kv0.close()
    lens = [mp * 16, mp * 16 - 37]
    kv, f = make_ctx(w, max_position=mp * 16 + 16)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, lens, extra_pages=1)
        bt = np.pad(bt, ((0, 0), (0, mp - bt.shape[1])))
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        qn = gen.make_queries(B, w.H, w.d_h, seed=7)
        q = bf16_tensor(qn)
        btd = torch.from_numpy(np.ascontiguousarray(bt)).cuda()
        sl = torch.tensor(np.asarray(lens, np.int32)).cuda()
        assert S.starkv_workspace_bytes(kv.ctx, S.OP_DECODE, B, mp) == ws
        ref = kv.decode(lc, q, btd, sl).float().cpu().numpy()
        want = O.decode(oc, qn, f.B_k, f.B_v, bt, lens)
        check_attention(ref, want, "workspace decode")
        for call in range(2):
            out = torch.full_like(q, float("nan"))
            S.starkv_decode_attn_noalloc(kv.ctx, lc.struct, q, btd, sl, out)
            got = out.float().cpu().numpy()
            check_attention(got, want, f"no-allocation decode, call {call}")
            assert np.abs(got - ref).max() <= ATOL_MAX
        assert kv.status() == 0
    finally:
        kv.close()


def test_noalloc_limit_is_the_tensor_core_workspace():
    """A shape whose CUDA-core partials would fit in 16 MiB but whose
    tensor-core workspace (score rows, query images, partials) does not is
    rejected: the documented limit is starkv_workspace_bytes, not the partials."""
    S = skv()
    w = gen.workload(1)
    kv, _ = make_ctx(w, max_position=64)
    try:
        B, mp = 64, 2048
        assert _simt_workspace(B, w.H, w.R, mp) <= SCRATCH
        assert S.starkv_workspace_bytes(kv.ctx, S.OP_DECODE, B, mp) > SCRATCH
        lc = kv.new_cache(1)
        q = torch.zeros((B, w.H, w.d_h), dtype=torch.bfloat16, device="cuda")
        bt = torch.zeros((B, mp), dtype=torch.int32, device="cuda")
        sl = torch.ones(B, dtype=torch.int32, device="cuda")
        with pytest.raises(S.StarKVError) as e:
            S.starkv_decode_attn_noalloc(kv.ctx, lc.struct, q, bt, sl, torch.empty_like(q))
        assert e.value.code == S.ERR_UNSUPPORTED_SHAPE
    finally:
        kv.close()
