"""bench.py's decode, stream and prefill legs run end to end on the CPU against
stand-ins for CUDA (events, streams, pinned memory) and for the library's
device entry points.

The stand-ins check what reaches the C ABI: the argument count and the pointer
types of every call, and, for the stream leg, that step i of a run appends and
decodes stream step i mod n: its hidden states, slots, query and lengths.
Layout queries go to the real library (host-only).  The same legs also run
as two gloo ranks (the bench's N > 1 path with gloo in place of NCCL): each rank
runs its own batch, rank 0 alone prints, and the job rate is the tokens of all
ranks over the slowest rank's time.  Nothing here measures anything; it guards
the bench's plumbing.
"""
import contextlib
import ctypes
import io
import json
import os
import socket
import time

import pytest
import torch
import torch.multiprocessing as mp

import bench
from harness import gen
from rank_mixed_precision_b200 import starkv as S


class _Event:
    def __init__(self, enable_timing=False):
        self.t = None

    def record(self, *a):
        self.t = time.perf_counter()

    def elapsed_time(self, other):
        return max(1e-6, (other.t - self.t) * 1e3)

    def synchronize(self):
        pass


class _Stream:
    cuda_stream = 0


class _Lib:
    """Device entry points recorded; everything else goes to the real library."""

    def __init__(self, real, log):
        self.real, self.log = real, log

    def __getattr__(self, name):
        return getattr(self.real, name)

    def starkv_append(self, *a):
        assert len(a) == 7
        _, _, x, sl, n, lat, _ = a
        assert isinstance(x, ctypes.c_void_p) and x.value and isinstance(sl, ctypes.c_void_p) and sl.value
        assert int(n) >= 1 and lat is None
        self.log.append(("append", x.value, sl.value))
        return 0

    def starkv_decode_attn(self, *a):
        assert len(a) == 11
        _, _, q, bt, ln, B, mp, out, ws, wsb, _ = a
        assert all(isinstance(p, ctypes.c_void_p) and p.value for p in (q, bt, ln, out, ws))
        assert int(B) >= 1 and int(mp) >= 1 and int(wsb) > 0
        self.log.append(("decode", q.value, ln.value))
        return 0

    def starkv_prefill_attn(self, *a):
        assert len(a) == 14
        _, _, q, cu, bt, ln, B, mp, tq, mq, out, ws, wsb, _ = a
        assert all(isinstance(p, ctypes.c_void_p) and p.value for p in (q, cu, bt, ln, out, ws))
        assert int(B) >= 1 and int(mp) >= 1 and int(tq) >= int(B) and 1 <= int(mq) <= int(mp) * 16 and int(wsb) > 0
        self.log.append(("prefill", q.value, int(tq), int(mq)))
        return 0

    def starkv_last_error(self):
        return b""


class _KV:
    """StarKV without a device: caches in host memory, fills recorded."""

    def __init__(self, log):
        self.log = log

    def __call__(self, cfg, *factors, stream=None):
        self.cfg, self.ctx = cfg, ctypes.c_void_p(1)
        return self

    def new_cache(self, n_pages):
        return S.LatentCache(self.cfg, n_pages, device="cpu")

    def append(self, cache, X, slots):
        assert X.dtype == torch.bfloat16 and X.dim() == 2 and X.is_contiguous()
        assert slots.dtype == torch.int64 and slots.shape == (X.shape[0],)
        assert 0 <= int(slots.min()) and int(slots.max()) < cache.n_pages * 16
        self.log.append(("fill", X.shape[0], slots.tolist()))

    def workspace(self, op, batch, max_pages, total_q=0):
        return torch.zeros(1 << 12, dtype=torch.uint8)

    def status(self):
        return 0


def _need_host(t, dtype, name, ndim=None):
    assert isinstance(t, torch.Tensor) and t.dtype == dtype and t.is_contiguous(), name
    assert ndim is None or t.dim() == ndim, name


def _install(monkeypatch):
    """Stand-ins for CUDA and the device entry points, plus small workloads."""
    log = []
    real_device = torch.device
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a: None)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a: _Stream())
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    monkeypatch.setattr(torch, "device", lambda *a, **k: real_device("cpu"))
    lib = _Lib(S.lib(), log)
    monkeypatch.setattr(S, "lib", lambda: lib)
    monkeypatch.setattr(S, "StarKV", _KV(log))
    monkeypatch.setattr(S, "_need", _need_host)
    small = {
        "dry_stream": gen.shrink(gen.workload("longchat7b_stream_b1_t32768_s128"), name="dry_stream", H=4, h_kv=4,
                                 d_h=64, hidden=256, r_k=16, R=64, batch=2, ctx=70, steps=9),
        "dry_decode": gen.shrink(gen.workload("longchat7b_decode_b16_t4096"), name="dry_decode", H=4, h_kv=4,
                                 d_h=64, hidden=256, r_k=16, R=64, batch=3, ctx=50),
        "dry_prefill": gen.shrink(gen.workload("longchat7b_prefill_b4_t30720_c2048"), name="dry_prefill", H=4,
                                  h_kv=4, d_h=64, hidden=256, r_k=16, R=64, batch=2, ctx=40, chunk=24),
    }
    monkeypatch.setattr(gen, "WORKLOADS", {**gen.WORKLOADS, **small})
    states = []
    init = bench.StreamState.__init__

    def recording_init(self, *a, **k):
        init(self, *a, **k)
        states.append(self)

    monkeypatch.setattr(bench.StreamState, "__init__", recording_init)
    return log, states


@pytest.fixture
def dry(monkeypatch):
    return _install(monkeypatch)


def _run(argv):
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main(argv)
    return json.loads(buf.getvalue().strip().splitlines()[-1])


def test_stream_leg_walks_the_stream_in_order(dry):
    log, states = dry
    steps, warm = 25, 3
    line = _run(["--workload", "dry_stream", "--steps", str(steps), "--warmup", str(warm), "--no-cpu-baseline",
                 "--only", "--sustain-seconds", "0"])
    st = states[-1]
    n, L0 = st.n, st.L0
    # every replica source: context [0, L0) in chunks, then each stream token alone, in order
    fills = [e for e in log if e[0] == "fill"]
    assert sum(e[1] for e in fills) == int(L0.sum()) + n * len(L0)
    assert [e[2] for e in fills[-n:]] == [st.slots_np[s].tolist() for s in range(n)]
    apps = [e for e in log if e[0] == "append"]
    decs = [e for e in log if e[0] == "decode"]
    assert len(apps) == len(decs) == 2 * (warm + steps)   # device-resident leg, then end to end
    for i in range(steps):
        s = i % n
        assert apps[warm + i][1:] == (st.X[s].data_ptr(), st.slots[s].data_ptr())
        assert decs[warm + i][1:] == (st.q[s].data_ptr(), st.lens[s].data_ptr())
    for s in range(n):
        for b in range(len(L0)):
            pos = int(L0[b]) + s
            assert st.lens_np[s, b] == pos + 1
            assert st.slots_np[s, b] == st.bt_np[b, pos // 16] * 16 + pos % 16
    assert line["steps"] == steps and line["warmup"] == warm
    assert line["config"]["ctx"] == f"{int(L0.max())} -> {int(L0.max()) + n}"
    assert line["e2e"]["h2d_bytes_per_step"] > 0 and line["e2e"]["d2h_bytes_per_step"] == 2 * 4 * 64 * 2
    assert line["gpu_launches"] == 6 * steps and line["roofline"]["traffic"] is None


def test_decode_leg_line_has_the_contract_keys(dry):
    log, _ = dry
    line = _run(["--workload", "dry_decode", "--steps", "7", "--warmup", "3", "--no-cpu-baseline", "--only",
                 "--sustain-seconds", "0.01"])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks", "sustained"):
        assert k in line, k
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic", "spec_gbs", "frac_of_spec"):
        assert k in line["roofline"], k
    assert line["roofline"]["frac_of_spec"] == pytest.approx(line["roofline"]["achieved"] / 8000.0)
    assert line["config"]["workload"] == "dry_decode" and line["n_gpus"] == 1
    # timed steps and the repeat pass: every one through the C ABI, then the end-to-end leg
    sus = line["sustained"]["steps"]
    assert sus >= 32 and sum(1 for e in log if e[0] == "decode") == 2 * (3 + 7) + sus


def test_prefill_leg_line_counts_its_launches_and_copies(dry):
    log, _ = dry
    steps, warm = 4, 3
    line = _run(["--workload", "dry_prefill", "--steps", str(steps), "--warmup", str(warm), "--no-cpu-baseline",
                 "--only", "--sustain-seconds", "0"])
    pre = [e for e in log if e[0] == "prefill"]
    assert len(pre) == 2 * (warm + steps)                  # device-resident leg, then end to end
    assert all(e[2] == 2 * 24 and e[3] == 24 for e in pre)
    # 48 appended tokens take the split-K append (2 kernels); the prefill is re-expansion + attention
    assert line["gpu_launches"] == (2 + 2) * steps
    assert line["e2e"]["unit"] == "TFLOP/s" and line["e2e"]["d2h_bytes_per_step"] == 48 * 4 * 64 * 2
    assert line["e2e"]["h2d_bytes_per_step"] >= 48 * 256 * 2 + 48 * 8 + 48 * 4 * 64 * 2


def test_prefill_reference_arm_reports_the_prefill_metric():
    w = gen.shrink(gen.workload("longchat7b_prefill_b4_t30720_c2048"), H=4, h_kv=4, d_h=64, hidden=256, r_k=16,
                   R=64, batch=2, ctx=40, chunk=24)

    class A:
        seed, steps, warmup = 0, 2, 1

    line = bench._run_reference_prefill(A, w, 1)
    assert line["metric"] == "prefill TFLOP/s (algorithmic)" and line["unit"] == "TFLOP/s"
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["value"] == line["value"] and line["e2e"]["h2d_bytes_per_step"] == 0


def _rank_worker(rank, world, port, workload, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    patch = pytest.MonkeyPatch()
    try:
        log, _ = _install(patch)
        init = bench.init_dist
        patch.setattr(bench, "init_dist", lambda world, backend: init(world, "gloo"))
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.main(["--workload", workload, "--steps", "6", "--warmup", "3", "--no-cpu-baseline",
                        "--gpus", str(world), "--sustain-seconds", "0"])
        q.put((rank, buf.getvalue(), sum(1 for e in log if e[0] == "decode")))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, "error", repr(e)))
    finally:
        patch.undo()


@pytest.mark.parametrize("workload", ["dry_decode", "dry_stream"])
def test_two_gloo_ranks_run_the_bench_and_rank0_prints_the_job_line(workload):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    procs = [ctx.Process(target=_rank_worker, args=(r, world, port, workload, q)) for r in range(world)]
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
        assert res[r][2] == 2 * (3 + 6)             # every rank runs its own batch: no work is skipped
    assert res[1][1].strip() == ""                   # only rank 0 prints
    line = json.loads(res[0][1].strip().splitlines()[-1])
    assert line["n_gpus"] == 2 and line["scaling"] == "weak" and line["steps"] == 6
    w = gen.shrink(gen.workload("longchat7b_decode_b16_t4096"), H=4, h_kv=4, d_h=64, hidden=256, r_k=16, R=64,
                   batch=3, ctx=50) if workload == "dry_decode" else None
    if w is not None:
        # whole-job rate: tokens of both ranks over the slowest rank's time
        tokens = 2 * 6 * int(gen.make_seq_lens(w).sum())
        assert line["value"] == pytest.approx(tokens / (line["ms_per_step"] * 6 / 1e3), rel=1e-9)


def test_headline_line_carries_a_record_per_workload(dry, monkeypatch):
    log, _ = dry
    monkeypatch.setattr(bench, "SUBRECORDS", ["dry_decode", "dry_stream", "dry_prefill"])
    line = _run(["--workload", "dry_decode", "--steps", "4", "--warmup", "3", "--no-cpu-baseline",
                 "--sustain-seconds", "0"])
    recs = line["workloads"]
    assert set(recs) == {"dry_stream", "dry_prefill"}          # the headline is not repeated
    for name, r in recs.items():
        for k in ("metric", "value", "unit", "roofline", "e2e", "clocks", "gpu_launches", "config"):
            assert k in r, (name, k)
        assert r["config"]["workload"] == name
    assert recs["dry_stream"]["steps"] == 9                    # the stream walks all its steps
    assert recs["dry_prefill"]["roofline"]["bound"] == "tensor"


def test_gpus_flag_starts_the_ranks_itself(monkeypatch):
    calls = []
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(bench.subprocess, "call", lambda cmd: calls.append(cmd) or 0)
    bench.main(["--gpus", "2", "--steps", "5", "--warmup", "3"])
    (cmd,) = calls
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=2" in cmd and "--master-addr=127.0.0.1" in cmd and "--nnodes=1" in cmd
    assert cmd[-6:] == ["--gpus", "2", "--steps", "5", "--warmup", "3"]
    assert cmd[-7].endswith("bench.py")


def test_gpus_flag_must_match_the_launched_ranks(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.main(["--gpus", "4", "--steps", "5", "--warmup", "3"])


def test_traffic_is_reported_only_for_the_captured_kernels(tmp_path, monkeypatch):
    table = tmp_path / "t.txt"
    d = bench.kernel_source_digest()
    table.write_text(f"# workload what bytes digest\nwl decode_call 123456 {d}\nwl2 decode_call 7 0000000000000000\n")
    monkeypatch.setattr(bench, "TRAFFIC_TABLE", str(table))
    assert bench.dram_traffic("wl", "decode_call") == (123456, "ncu capture of the current kernels")
    assert bench.dram_traffic("wl2", "decode_call")[0] is None
    assert "changed" in bench.dram_traffic("wl2", "decode_call")[1]
    assert bench.dram_traffic("other", "decode_call")[0] is None
