"""Sequence sharding plumbing on CPU: two gloo ranks each hold one slice of a
sequence's context, run the sharded decode step (slice attention, one
all-gather, merge) through rank_mixed_precision_b200.seqshard, and must reach
the whole-sequence oracle decode.  The device entry points are stood in for by
the fp64 oracle on host tensors (the plumbing is under test, not the kernels)."""
import math
import os
import socket
import types

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle as O
from harness import gen
from rank_mixed_precision_b200 import seqshard


def test_token_ranges_cover_and_balance():
    for n in (0, 1, 7, 32768, 32769):
        for world in (1, 2, 3, 8):
            r = seqshard.token_ranges(n, world)
            assert len(r) == world and r[0][0] == 0 and r[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(r[:-1], r[1:]))
            sizes = [hi - lo for lo, hi in r]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        seqshard.token_ranges(10, 0)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        w = gen.workload(0)
        cfg = O.config_of(w)
        n = 260
        f = gen.make_factors(w)
        zk, zv = gen.make_latents(w, n)
        lo, hi = seqshard.slice_of(n, rank, world)
        sbt, sp = gen.make_block_table([hi - lo], seed=rank + 1)
        cache = O.new_cache(cfg, sp)
        O.write_latents(cache, gen.slots_for(sbt, 0, np.arange(hi - lo)), zk[lo:hi], zv[lo:hi])
        qn = gen.make_queries(1, w.H, w.d_h, seed=2)
        S = seqshard.S
        calls = {}

        def slice_stand_in(ctx, cache_struct, q, bt, lens, pos0, qpos, o, ml, ws, stream=None):
            ro, rm, rl = O.decode_slice(cache_struct, qn, f.B_k, f.B_v, bt.numpy(), lens.tolist(), pos0.tolist(),
                                        qpos.tolist())
            o.copy_(torch.from_numpy(ro))
            ml[..., 0] = torch.from_numpy(rm * (1.0 / math.log(2.0)))   # log2 units, as the library
            ml[..., 1] = torch.from_numpy(rl)
            calls["slice"] = (int(lens[0]), int(pos0[0]), int(qpos[0]))

        def merge_stand_in(ctx, o_parts, ml_parts, out, stream=None):
            m = ml_parts[..., 0].numpy() * math.log(2.0)
            out.copy_(torch.from_numpy(O.merge_slices(o_parts.numpy(), m, ml_parts[..., 1].numpy())))
            calls["merge"] = tuple(o_parts.shape)

        S_patch = types.SimpleNamespace(starkv_decode_attn_slice=slice_stand_in, starkv_merge_slices=merge_stand_in)
        seqshard.S = S_patch
        plan = seqshard.SlicePlan([n], rank, world, device="cpu")
        kv = types.SimpleNamespace(ctx=None)
        lc = types.SimpleNamespace(struct=cache)
        out = seqshard.decode_sharded(kv, lc, torch.zeros((1, w.H, w.d_h), dtype=torch.float64),
                                      torch.from_numpy(sbt), plan, workspace=None)
        bt, n_pages = gen.make_block_table([n])
        whole = O.new_cache(cfg, n_pages)
        O.write_latents(whole, gen.slots_for(bt, 0, np.arange(n)), zk, zv)
        ref = O.decode(whole, qn, f.B_k, f.B_v, bt, [n])
        err = float(np.abs(out.numpy() - ref).max())
        q.put((rank, err, calls))
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent
        q.put((rank, "error", repr(e)))


def test_two_gloo_ranks_merge_their_slices_into_the_whole_decode():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        item = q.get(timeout=180)
        res[item[0]] = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert res[r][1] != "error", res[r]
        assert res[r][1] < 1e-6, res[r]          # the exchanged rows are fp32
        lo, hi = seqshard.slice_of(260, r, world)
        assert res[r][2]["slice"] == (hi - lo, lo, 259)
        assert res[r][2]["merge"] == (world, 1, 4, 64)
