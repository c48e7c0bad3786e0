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

from _cases import ATOL_MAX, REL_L2, bf16_tensor, make_ctx, oracle_cache, skv, upload

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
        for call in range(2):           # the scratch keeps the previous call's contents
            out = torch.full_like(q, float("nan"))
            S.starkv_decode_attn_noalloc(kv.ctx, lc.struct, q, btd, sl, out)
            got = out.float()
            assert torch.isfinite(got).all(), f"call {call}: non-finite output"
            err = (got - ref).abs().max().item()
            rel = (torch.linalg.norm(got - ref) / torch.linalg.norm(ref).clamp_min(1e-30)).item()
            assert err <= ATOL_MAX and rel <= REL_L2, f"call {call}: max-abs {err:.3e} rel-L2 {rel:.3e}"
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
