"""Sequence sharding on one GPU: the context of a sequence split into slices,
each slice in its own cache (as each rank would hold it), decoded with
starkv_decode_attn_slice and merged with starkv_merge_slices, against the fp64
oracle (whole-sequence decode and per-slice statistics) and against the
ordinary decode of the whole sequence.  Ranks are emulated by calls in turn on
one GPU; no kernel waits on another."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from harness import gen

from _cases import ATOL_MAX, bf16_tensor, check_attention, make_ctx, skv, upload

pytestmark = pytest.mark.gpu


def _caches(w, n, cuts, seed=0):
    cfg = O.config_of(w)
    zk, zv = gen.make_latents(w, n, seed)
    bt, n_pages = gen.make_block_table([n], seed)
    whole = O.new_cache(cfg, n_pages)
    O.write_latents(whole, gen.slots_for(bt, 0, np.arange(n)), zk, zv)
    slices = []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        sbt, sp = gen.make_block_table([max(hi - lo, 1)], seed + lo + 1)
        c = O.new_cache(cfg, sp)
        if hi > lo:
            O.write_latents(c, gen.slots_for(sbt, 0, np.arange(hi - lo)), zk[lo:hi], zv[lo:hi])
        slices.append((c, sbt, sp, lo, hi))
    return whole, bt, n_pages, slices


@pytest.mark.parametrize("wi,n,cuts", [(0, 700, [0, 250, 250, 513, 700]), (1, 1500, [0, 600, 1100, 1500]),
                                       (3, 2000, [0, 1000, 1999, 2000])], ids=["tiny", "longchat", "llama3gqa"])
def test_sharded_decode_matches_oracle_and_whole_decode(wi, n, cuts):
    S = skv()
    w = gen.workload(wi)
    kv, f = make_ctx(w, max_position=n + 16)
    try:
        whole, bt, n_pages, slices = _caches(w, n, cuts)
        qn = gen.make_queries(1, w.H, w.d_h, seed=11)
        q = bf16_tensor(qn)
        o_parts, ml_parts = [], []
        for c, sbt, sp, lo, hi in slices:
            lc = kv.new_cache(sp)
            upload(lc, c)
            o = torch.full((1, w.H, w.d_h), float("nan"), dtype=torch.float32, device="cuda")
            ml = torch.full((1, w.H, 2), float("nan"), dtype=torch.float32, device="cuda")
            i32 = lambda v: torch.tensor([v], dtype=torch.int32, device="cuda")
            S.starkv_decode_attn_slice(kv.ctx, lc.struct, q, torch.from_numpy(sbt).cuda(), i32(hi - lo), i32(lo),
                                       i32(n - 1), o, ml, kv.workspace(S.OP_DECODE, 1, sbt.shape[1]))
            assert kv.status() == 0
            ro, rm, rl = O.decode_slice(c, qn, f.B_k, f.B_v, sbt, [hi - lo], [lo], [n - 1])
            got_ml = ml.cpu().numpy()[0]
            if hi > lo:
                check_attention(o.cpu().numpy(), ro, f"slice [{lo}, {hi})")
                # statistics: m in log2 units on the GPU; l within the fp16-operand tolerance
                np.testing.assert_allclose(got_ml[:, 0] * math.log(2.0), rm[0], atol=2e-2, rtol=0)
                np.testing.assert_allclose(got_ml[:, 1], rl[0], rtol=2e-2, atol=0)
            else:
                assert np.all(got_ml[:, 0] == -np.inf) and np.all(got_ml[:, 1] == 0)
                assert np.all(o.cpu().numpy() == 0)
            o_parts.append(o)
            ml_parts.append(ml)
        out = torch.empty_like(q)
        S.starkv_merge_slices(kv.ctx, torch.stack(o_parts).contiguous(), torch.stack(ml_parts).contiguous(), out)
        got = out.float().cpu().numpy()
        ref = O.decode(whole, qn, f.B_k, f.B_v, bt, [n])
        check_attention(got, ref, "merged slices")
        # and against the ordinary decode of the whole sequence on the GPU
        lw = kv.new_cache(n_pages)
        upload(lw, whole)
        plain = kv.decode(lw, q, torch.from_numpy(bt).cuda(), torch.tensor([n], dtype=torch.int32).cuda())
        assert np.abs(plain.float().cpu().numpy() - got).max() <= ATOL_MAX
        assert kv.status() == 0
    finally:
        kv.close()


def test_slice_positions_beyond_the_rope_table_set_status():
    S = skv()
    w = gen.workload(0)
    kv, f = make_ctx(w, max_position=300)
    try:
        whole, bt, n_pages, slices = _caches(w, 200, [0, 200])
        c, sbt, sp, lo, hi = slices[0]
        lc = kv.new_cache(sp)
        upload(lc, c)
        q = bf16_tensor(gen.make_queries(1, w.H, w.d_h))
        o = torch.zeros((1, w.H, w.d_h), dtype=torch.float32, device="cuda")
        ml = torch.zeros((1, w.H, 2), dtype=torch.float32, device="cuda")
        i32 = lambda v: torch.tensor([v], dtype=torch.int32, device="cuda")
        # 200 tokens from position 150 run past max_position 300
        S.starkv_decode_attn_slice(kv.ctx, lc.struct, q, torch.from_numpy(sbt).cuda(), i32(200), i32(150), i32(299),
                                   o, ml, kv.workspace(S.OP_DECODE, 1, sbt.shape[1]))
        assert kv.status() & S.DEV_BAD_SEQ_LEN
    finally:
        kv.close()
