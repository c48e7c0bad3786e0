"""Decode with the attention block's output projection (starkv_decode_attn_out)
against the fp64 oracle: y = sum_h o_h W_o,h ([Review] Algorithm 2 steps 7-8,
eq. 12)."""
import numpy as np
import pytest
import torch

import oracle as O
from harness import gen

from _cases import bf16_tensor, check_attention, make_ctx, oracle_cache, skv, upload

pytestmark = pytest.mark.gpu


def _w_o(w, model, seed=21):
    rng = np.random.default_rng(seed)
    return gen.to_bf16((rng.standard_normal((w.H * w.d_h, model)) / np.sqrt(w.H * w.d_h)).astype(np.float32))[0]


@pytest.mark.parametrize("wi,lens,model", [(0, [256, 17, 1, 0], 256), (1, [300, 1000, 64], 4096),
                                           (3, [700, 1500, 33], 4096)], ids=["tiny", "longchat", "llama3gqa"])
def test_decode_out_matches_oracle(wi, lens, model):
    S = skv()
    w = gen.workload(wi)
    kv, f = make_ctx(w, max_position=max(lens) + 16)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, lens, extra_pages=1)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        Wo = _w_o(w, model)
        S.starkv_set_output_projection(kv.ctx, bf16_tensor(Wo))
        qn = gen.make_queries(len(lens), w.H, w.d_h)
        btd = torch.from_numpy(bt).cuda()
        sl = torch.tensor(np.asarray(lens, np.int32)).cuda()
        y = torch.full((len(lens), model), float("nan"), dtype=torch.bfloat16, device="cuda")
        ws = kv.workspace(S.OP_DECODE_OUT, len(lens), bt.shape[1])
        S.starkv_decode_attn_out(kv.ctx, lc.struct, bf16_tensor(qn), btd, sl, y, ws)
        assert kv.status() == 0
        ref = O.decode_out(oc, qn, f.B_k, f.B_v, Wo, bt, lens)
        check_attention(y.float().cpu().numpy(), ref, "decode with output projection")
    finally:
        kv.close()


def test_decode_out_batch_above_64_rows():
    # the output GEMM runs in 64-row blocks
    S = skv()
    w = gen.workload(0)
    lens = [40 + 3 * i for i in range(70)]
    kv, f = make_ctx(w, max_position=max(lens) + 16)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, lens)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        Wo = _w_o(w, 128)
        S.starkv_set_output_projection(kv.ctx, bf16_tensor(Wo))
        qn = gen.make_queries(len(lens), w.H, w.d_h)
        y = torch.empty((len(lens), 128), dtype=torch.bfloat16, device="cuda")
        S.starkv_decode_attn_out(kv.ctx, lc.struct, bf16_tensor(qn), torch.from_numpy(bt).cuda(),
                                 torch.tensor(np.asarray(lens, np.int32)).cuda(), y,
                                 kv.workspace(S.OP_DECODE_OUT, len(lens), bt.shape[1]))
        assert kv.status() == 0
        check_attention(y.float().cpu().numpy(), O.decode_out(oc, qn, f.B_k, f.B_v, Wo, bt, lens), "70 rows")
    finally:
        kv.close()


def test_decode_out_needs_an_output_projection():
    S = skv()
    w = gen.workload(0)
    kv, f = make_ctx(w, max_position=64)
    try:
        with pytest.raises(S.StarKVError) as e:
            S.starkv_workspace_bytes(kv.ctx, S.OP_DECODE_OUT, 1, 1)
        assert e.value.code == S.ERR_INVALID_ARG
        lc = kv.new_cache(1)
        q = torch.zeros((1, w.H, w.d_h), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(S.StarKVError):
            S.starkv_decode_attn_out(kv.ctx, lc.struct, q, torch.zeros((1, 1), dtype=torch.int32, device="cuda"),
                                     torch.ones(1, dtype=torch.int32, device="cuda"),
                                     torch.empty((1, 64), dtype=torch.bfloat16, device="cuda"),
                                     torch.empty(256, dtype=torch.uint8, device="cuda"))
    finally:
        kv.close()
