"""Multi-rank host logic of bench.py on CPU ranks (gloo, world size 2).

Decode shards by sequence with no data-path collective: each rank owns its own
batch (weak scaling) and the only cross-rank steps are the timing barrier, the
maximum of the per-rank times and the sum of the per-rank token counts.  These
tests run those steps on two gloo ranks.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    try:
        dist = bench.init_dist(world, "gloo")
        r, w, local = bench.dist_env()
        assert (r, w, local) == (rank, world, rank)
        bench.barrier(world)
        # per-rank time and token counts differ; the job rate uses the slowest time
        ms = 10.0 * (rank + 1)
        units = 1000.0 * (rank + 1)
        mx = bench.max_over_ranks(ms, world)
        total = bench.sum_over_ranks(units, world)
        rate, ms_max = bench.job_throughput(units, ms, world)
        # the reference arm runs on rank 0 only; the other ranks do no work
        ref = bench.run_reference(None, None, rank, world) if rank != 0 else "rank0"
        q.put((rank, mx, total, rate, ms_max, ref))
        bench.barrier(world)
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, "error", repr(e)))


def test_two_gloo_ranks_agree_on_max_time_and_total_tokens():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        item = q.get(timeout=120)
        res[item[0]] = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert res[r][1] != "error", res[r]
        _, mx, total, rate, ms_max, ref = res[r]
        assert mx == pytest.approx(20.0)
        assert total == pytest.approx(3000.0)
        assert ms_max == pytest.approx(20.0)
        assert rate == pytest.approx(3000.0 / 0.020)
    assert res[1][5] is None


@pytest.mark.parametrize("batch,world", [(16, 2), (7, 2), (1, 2), (5, 4)])
def test_strong_sharding_partitions_the_batch(batch, world):
    owned = [bench.shard_sequences(batch, r, world, "strong")[0] for r in range(world)]
    flat = [b for o in owned for b in o]
    assert sorted(flat) == list(range(batch))
    assert len(set(flat)) == batch


def test_weak_sharding_gives_every_rank_the_full_batch():
    for r in range(3):
        owned, _ = bench.shard_sequences(16, r, 3, "weak")
        assert owned == list(range(16))


def test_single_rank_helpers_need_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.sum_over_ranks(2.0, 1) == 2.0
    rate, ms = bench.job_throughput(500.0, 250.0, 1)
    assert ms == 250.0 and rate == pytest.approx(2000.0)
    bench.barrier(1)
