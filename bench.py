"""Benchmark: decode context-tokens/s and achieved HBM GB/s of STAR-KV latent-cache attention.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl starkv|reference] [--workload NAME]

One step = one pass of the hot path over one batch.  Decode workloads: append
one new token per sequence (project, rotate, quantise, pack), then batched
single-query attention over the packed cache (dequantise, re-expand and RoPE
keys, online softmax, P Z_v in the latent, split merge, B_v projection).
Prefill workload: append a chunk of tokens, then causal attention of the
chunk's queries over the whole cache.

Default (headline) workload: Llama-3-8B-shaped GQA decode layer, 32 query
heads over 8 KV heads, d_h 128, r_k 64, R 512, batch 32, ragged contexts
U[4096, 8192], 16-token pages.  At N = 1 the line also carries one record per
other workload (LongChat-7B-shaped decode at batch 16 x 4096, the 128-step
single-stream run from 32768 tokens, and the chunked prefill), each with its
own roofline, end-to-end figure, clocks and CPU oracle baseline.  Inputs are
seeded and synthetic (no weights or datasets).

With --gpus N > 1 outside torchrun, the bench starts N ranks itself through
torch.distributed.run (one process per GPU).  Every rank runs its own batch of
independent sequences (weak scaling, no collective on the data path); the
timing is the maximum over ranks.  The reference arm times the fp64 CPU oracle
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from harness import gen  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
SPEC_HBM_GBS = 8000.0          # B200 HBM3e bandwidth as specified (DGX figure)
FALLBACK_HBM_GBS = 6650.0      # copy bandwidth measured earlier on this kind of GPU
FALLBACK_BF16_TFLOPS = 1590.0  # cuBLAS bf16 burst measured earlier on this kind of GPU
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0

HEADLINE = "llama3_8b_gqa_decode_b32_t4096to8192"
SUBRECORDS = ["longchat7b_decode_b16_t4096", "longchat7b_stream_b1_t32768_s128",
              "longchat7b_prefill_b4_t30720_c2048"]
CSRC = os.path.join(ROOT, "rank_mixed_precision_b200", "csrc")
TRAFFIC_TABLE = os.path.join(ROOT, "profiles", "dram_traffic.txt")


# ---------------------------------------------------------------------------
# distributed plumbing (timing only; no data-path collective)
# ---------------------------------------------------------------------------
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_throughput(units_local: float, ms_local: float, world: int, device=None):
    """Whole-job rate: the units every rank processed over the slowest rank's time."""
    ms_max = max_over_ranks(ms_local, world, device)
    units = sum_over_ranks(units_local, world, device)
    return units / (ms_max / 1e3), ms_max


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def shard_sequences(batch: int, rank: int, world: int, scaling: str = "weak"):
    """Sequences owned by `rank`: weak scaling gives every rank its own full batch."""
    if scaling == "weak":
        return list(range(batch)), rank
    per = (batch + world - 1) // world
    return list(range(rank * per, min(batch, (rank + 1) * per))), 0


def free_port() -> int:
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launch_ranks(n: int, argv) -> int:
    """Run this script as n ranks (one process per GPU) under torch.distributed.run."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={free_port()}", os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


# ---------------------------------------------------------------------------
# clocks: sampled by a host thread from warm-up to the end of the repeat pass
# ---------------------------------------------------------------------------
# NVML clock event reason bits
_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}
_IDLE = 0x1


class ClockSampler:
    """Samples SM clock, its maximum, power and throttle reasons every ~10 ms
    (NVML, read-only queries; nvidia-smi when NVML is unavailable).  mark()
    records the start of a named phase so a summary covers chosen phases."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active")

    def __init__(self, gpu_index: int, period_s: float = 0.01):
        self.idx, self.period = gpu_index, period_s
        self.samples = []           # (t, sm_mhz, max_mhz, reasons_mask, power_w)
        self.marks = {}
        self._stop = threading.Event()
        self._thread = None
        self.source = None

    def _nvml_loop(self, nv, h):
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                rs = get(h)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1e3
                self.samples.append((time.perf_counter(), float(sm), float(mx), int(rs), float(pw)))
            except Exception:
                pass
            self._stop.wait(self.period)

    def _smi_loop(self, proc):
        for line in proc.stdout:
            if self._stop.is_set():
                break
            p = [x.strip() for x in line.split(",")]
            if len(p) < 5:
                continue
            try:
                self.samples.append((time.perf_counter(), float(p[1]), float(p[2]), int(p[4], 16),
                                     float(p[3])))
            except ValueError:
                continue

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self._physical_index())
            self.source = "nvml"
            self._thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
        except Exception:
            self.proc = None
            try:
                self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self._physical_index()), f"--query-gpu={self.Q}",
                                              "--format=csv,noheader,nounits", "-lms", "50"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi"
                self._thread = threading.Thread(target=self._smi_loop, args=(self.proc,), daemon=True)
            except Exception:
                self._thread = None
        if self._thread is not None:
            self._thread.start()
            t0 = time.perf_counter()
            while not self.samples and time.perf_counter() - t0 < 5.0:  # the sampler sees the run from its start
                time.sleep(0.005)
        self.mark("start")
        return self

    def _physical_index(self) -> int:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            ids = [v.strip() for v in vis.split(",") if v.strip()]
            if self.idx < len(ids) and ids[self.idx].isdigit():
                return int(ids[self.idx])
        return self.idx

    def mark(self, name):
        self.marks[name] = time.perf_counter()

    def __exit__(self, *a):
        self.mark("end")
        self._stop.set()
        if getattr(self, "proc", None) is not None:
            self.proc.terminate()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self, since: str = "start", until: str = "end"):
        t0, t1 = self.marks.get(since, 0.0), self.marks.get(until, float("inf"))
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        busy = [s for s in win if not s[3] & _IDLE] or win
        if not busy:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        reasons = sorted({n for s in busy for bit, n in _REASONS.items() if s[3] & bit})
        return {"sm_mhz": statistics.median(s[1] for s in busy), "sm_max_mhz": max(s[2] for s in busy),
                "power_w_max": max(s[4] for s in busy), "reasons": reasons, "samples": len(busy),
                "source": self.source, "window_s": round(t1 - t0, 3) if t1 != float("inf") else None}


def sustained_pass(step, first: int, seconds: float, ms_hint: float = 0.0):
    """Steps back to back for at least `seconds` of device time (CUDA events on
    the launching stream); returns steps run and ms per step.  ms_hint (a step's
    time from the timed region) sizes the first batch of steps."""
    import torch
    chunk = 32 if ms_hint <= 0 else max(1, min(32, int(0.05 * seconds * 1e3 / ms_hint)))
    n, ms = 0, 0.0
    while ms < seconds * 1e3:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for k in range(chunk):
            step(first + n + k)
        b.record()
        b.synchronize()
        ms += a.elapsed_time(b)
        n += chunk
        chunk = min(chunk * 2, 4096)
    return n, ms / n


def sustained_record(n, ms_per_step, units_per_step, clocks, unit):
    rec = {"steps": n, "seconds": n * ms_per_step / 1e3, "ms_per_step": ms_per_step,
           "value": units_per_step / (ms_per_step / 1e3), "unit": unit}
    if clocks.get("sm_mhz"):
        rec["sm_mhz_median"] = clocks["sm_mhz"]
        rec["ms_x_mhz"] = ms_per_step * clocks["sm_mhz"]
    return rec


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """(sustained bf16 TFLOP/s, kind): the denominator for a kernel timed inside a long step."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        if "bf16_tflops_sustained" in d:
            return float(d["bf16_tflops_sustained"]), "measured, sustained"
        return float(d["bf16_tflops"]), "measured, burst"
    return FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback, sustained"


def kernel_source_digest() -> str:
    """Digest of the library's CUDA sources: DRAM traffic counted on one version
    of the kernels is reported only while the sources are unchanged."""
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            h.update(name.encode())
            h.update(open(os.path.join(CSRC, name), "rb").read())
    return h.hexdigest()[:16]


def dram_traffic(workload: str, what: str):
    """DRAM bytes (read + write) per call from the committed ncu summary table:
    lines `<workload> <what> <bytes> <source digest>`; None when the kernels
    changed after the capture or nothing was captured."""
    try:
        lines = open(TRAFFIC_TABLE).read().splitlines()
    except OSError:
        return None, "no capture"
    digest = kernel_source_digest()
    stale = False
    for ln in lines:
        p = ln.split()
        if len(p) >= 4 and not ln.startswith("#") and p[0] == workload and p[1] == what:
            if p[3] == digest:
                return int(p[2]), "ncu capture of the current kernels"
            stale = True
    return None, "kernels changed since the last capture" if stale else "no capture"


def pack_layout(tensors, align: int = 256):
    """Byte offsets that lay `tensors` out back to back in one buffer, each
    start rounded up to `align`, and the buffer's total size."""
    offs, total = [], 0
    for t in tensors:
        total = -(-total // align) * align
        offs.append(total)
        total += t.numel() * t.element_size()
    return offs, total


def packed_views(buf, offs, like):
    """Typed views of the 1-D uint8 `buf` at `offs`, shaped like `like`."""
    return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for o, t in zip(offs, like)]


def stream_schedule(seq_lens0, n_steps: int, block_table):
    """Long-context stream: at step s every sequence appends the token at
    position L0 + s and then decodes its context of L0 + s + 1 tokens.
    Returns (slots [n_steps, B] int64, seq_lens [n_steps, B] int32)."""
    L0 = np.asarray(seq_lens0, np.int64)
    steps = np.arange(n_steps, dtype=np.int64)
    slots = np.stack([gen.slots_for(block_table, b, L0[b] + steps) for b in range(L0.shape[0])], axis=1)
    lens = (L0[None, :] + steps[:, None] + 1).astype(np.int32)
    return slots.reshape(n_steps, L0.shape[0]), lens


# ---------------------------------------------------------------------------
# workload state on the GPU
# ---------------------------------------------------------------------------
def bytes_per_token(w) -> int:
    """Packed cache bytes per token from the library's own layout query."""
    from rank_mixed_precision_b200 import starkv as S
    cfg = S.make_config(w.H, w.h_kv, w.d_h, w.hidden, w.r_k, w.R, 16, w.top_fraction, w.rope_base)
    sz = S.starkv_cache_layout(cfg, 1)
    return (sz["k_codes_bytes"] + sz["v_codes_bytes"] + sz["k_meta_bytes"] + sz["v_meta_bytes"]) // 16


def decode_algorithmic_bytes(w, total_tokens: int, batch: int, max_pages: int) -> int:
    """What one decode call must move once: packed payload + metadata of every
    attended token, the bf16 up-projections B_k and B_v, q, out, block table and lengths."""
    factors = 2 * (w.h_kv * w.r_k * w.d_h + w.R * w.h_kv * w.d_h)
    io = 2 * 2 * batch * w.H * w.d_h + 4 * batch * max_pages + 4 * batch
    return total_tokens * bytes_per_token(w) + factors + io


class DecodeState:
    def __init__(self, w, seed, device, replicas):
        import torch
        from rank_mixed_precision_b200 import starkv as S
        self.S = S
        self.w = w
        bf = lambda a: torch.from_numpy(gen.bf16_bits(a).view(np.int16).copy()).view(torch.bfloat16).to(device)
        f = gen.make_factors(w, seed)
        self.seq_lens = gen.make_seq_lens(w, seed)
        B = w.batch
        mp = int(self.seq_lens.max()) + 16
        cfg = S.make_config(w.H, w.h_kv, w.d_h, w.hidden, w.r_k, w.R, mp, w.top_fraction, w.rope_base)
        self.kv = S.StarKV(cfg, bf(f.A_k), bf(f.A_v), bf(f.B_k), bf(f.B_v))
        bt, n_pages = gen.make_block_table(self.seq_lens, seed)
        self.bt_np = bt
        self.max_pages = bt.shape[1]
        self.n_pages = n_pages
        # fill the context [0, L-1) of every sequence with the library's own append
        self.caches = [self.kv.new_cache(n_pages) for _ in range(replicas)]
        chunk = 4096
        for b in range(B):
            L = int(self.seq_lens[b])
            for s0 in range(0, L - 1, chunk):
                n = min(chunk, L - 1 - s0)
                X = bf(gen.make_hidden(n, w.hidden, seed, name="X", sub=1000 * b + s0 // chunk))
                slots = torch.from_numpy(gen.slots_for(bt, b, np.arange(s0, s0 + n))).to(device)
                self.kv.append(self.caches[0], X, slots)
        torch.cuda.synchronize()
        for c in self.caches[1:]:
            for name in ("k_codes", "v_codes", "k_meta", "v_meta"):
                getattr(c, name).copy_(getattr(self.caches[0], name))
        # per-step inputs: one new token per sequence at position L-1, its query
        self.X_np = gen.make_hidden(B, w.hidden, seed, name="X_step")
        self.q_np = gen.make_queries(B, w.H, w.d_h, seed, name="q_step")
        self.slots_np = np.array([gen.slots_for(bt, b, [int(self.seq_lens[b]) - 1])[0] for b in range(B)],
                                 np.int64)
        self.X = bf(self.X_np)
        self.q = bf(self.q_np)
        self.slots = torch.from_numpy(self.slots_np).to(device)
        self.bt = torch.from_numpy(bt).to(device)
        self.sl = torch.from_numpy(self.seq_lens.astype(np.int32)).to(device)
        self.out = torch.empty_like(self.q)
        self.ws = self.kv.workspace(S.OP_DECODE, B, self.max_pages)
        st = self.kv.status()
        if st:
            raise RuntimeError(f"device status {st:#x} after cache fill")
        # pre-marshalled C-ABI arguments (the timed loop calls the C entry points directly)
        import ctypes
        self.lib = S.lib()
        vp = ctypes.c_void_p
        self.stream = vp(torch.cuda.current_stream().cuda_stream)
        self.args = []
        for c in self.caches:
            ref = ctypes.byref(c.struct)
            self.args.append((
                (self.kv.ctx, ref, vp(self.X.data_ptr()), vp(self.slots.data_ptr()), B, None, self.stream),
                (self.kv.ctx, ref, vp(self.q.data_ptr()), vp(self.bt.data_ptr()), vp(self.sl.data_ptr()), B,
                 self.max_pages, vp(self.out.data_ptr()), vp(self.ws.data_ptr()), self.ws.numel(), self.stream)))

    def step(self, i, ev=None):
        app, dec = self.args[i % len(self.args)]
        if self.lib.starkv_append(*app):
            raise RuntimeError(self.lib.starkv_last_error().decode())
        if ev is not None:
            ev[0].record()
        if self.lib.starkv_decode_attn(*dec):
            raise RuntimeError(self.lib.starkv_last_error().decode())
        if ev is not None:
            ev[1].record()


class StreamState:
    """Long-context stream (batch-1 style): run step i is stream step
    s = i mod n, which appends one token per sequence at position L0 + s and
    decodes the grown context of L0 + s + 1 tokens.

    Every replica is filled through all n stream positions before timing, the
    stream positions by the same single-token append a step issues, so a step's
    append rewrites identical bytes, and a decode, which reads only positions
    below its length, always sees exactly the stream's context."""

    def __init__(self, w, seed, device, replicas):
        import ctypes
        import torch
        from rank_mixed_precision_b200 import starkv as S
        self.S, self.w, self.n = S, w, w.steps
        bf = lambda a: torch.from_numpy(gen.bf16_bits(a).view(np.int16).copy()).view(torch.bfloat16).to(device)
        f = gen.make_factors(w, seed)
        B, n = w.batch, w.steps
        self.L0 = gen.make_seq_lens(w, seed)
        caps = self.L0.astype(np.int64) + n
        cfg = S.make_config(w.H, w.h_kv, w.d_h, w.hidden, w.r_k, w.R, int(caps.max()) + 16, w.top_fraction,
                            w.rope_base)
        self.kv = S.StarKV(cfg, bf(f.A_k), bf(f.A_v), bf(f.B_k), bf(f.B_v))
        bt, n_pages = gen.make_block_table(caps, seed)
        self.bt_np, self.max_pages = bt, bt.shape[1]
        self.slots_np, self.lens_np = stream_schedule(self.L0, n, bt)
        self.X_np = np.stack([gen.make_hidden(B, w.hidden, seed, name="X_step", sub=s) for s in range(n)])
        self.q_np = np.stack([gen.make_queries(B, w.H, w.d_h, seed, name="q_step", sub=s) for s in range(n)])
        self.X, self.q = bf(self.X_np), bf(self.q_np)
        self.slots = torch.from_numpy(self.slots_np).to(device)
        self.lens = torch.from_numpy(self.lens_np).to(device)
        self.bt = torch.from_numpy(bt).to(device)
        self.caches = [self.kv.new_cache(n_pages) for _ in range(replicas)]
        c0 = self.caches[0]
        chunk = 4096
        for b in range(B):
            L = int(self.L0[b])
            for s0 in range(0, L, chunk):
                m = min(chunk, L - s0)
                X = bf(gen.make_hidden(m, w.hidden, seed, name="X", sub=1000 * b + s0 // chunk))
                sl = torch.from_numpy(gen.slots_for(bt, b, np.arange(s0, s0 + m))).to(device)
                self.kv.append(c0, X, sl)
        for s in range(n):
            self.kv.append(c0, self.X[s], self.slots[s])
        torch.cuda.synchronize()
        for c in self.caches[1:]:
            for name in ("k_codes", "v_codes", "k_meta", "v_meta"):
                getattr(c, name).copy_(getattr(c0, name))
        self.out = torch.empty_like(self.q[0])
        self.ws = self.kv.workspace(S.OP_DECODE, B, self.max_pages)
        st = self.kv.status()
        if st:
            raise RuntimeError(f"device status {st:#x} after cache fill")
        # pre-marshalled C-ABI arguments (the timed loop calls the C entry points directly)
        self.lib = S.lib()
        vp = ctypes.c_void_p
        strm = vp(torch.cuda.current_stream().cuda_stream)
        self.refs = [ctypes.byref(c.struct) for c in self.caches]
        self.app = [(vp(self.X[s].data_ptr()), vp(self.slots[s].data_ptr()), B, None, strm) for s in range(n)]
        self.dec = [(vp(self.q[s].data_ptr()), vp(self.bt.data_ptr()), vp(self.lens[s].data_ptr()), B,
                     self.max_pages, vp(self.out.data_ptr()), vp(self.ws.data_ptr()), self.ws.numel(), strm)
                    for s in range(n)]

    def tokens(self, i) -> int:
        """Context tokens the decode of run step i attends to."""
        return int(self.lens_np[i % self.n].sum())

    def step(self, i, ev=None):
        s, ref = i % self.n, self.refs[i % len(self.refs)]
        x, sl, B, lat, strm = self.app[s]
        if self.lib.starkv_append(self.kv.ctx, ref, x, sl, B, lat, strm):
            raise RuntimeError(self.lib.starkv_last_error().decode())
        if ev is not None:
            ev[0].record()
        if self.lib.starkv_decode_attn(self.kv.ctx, ref, *self.dec[s]):
            raise RuntimeError(self.lib.starkv_last_error().decode())
        if ev is not None:
            ev[1].record()


class PrefillState:
    """Chunked prefill: each sequence holds `ctx` packed tokens; a step appends the
    next `chunk` tokens (their hidden states through the projection, rotation,
    quantiser and packer) and runs causal attention of those `chunk` queries over
    all ctx + chunk positions."""

    def __init__(self, w, seed, device):
        import torch
        from rank_mixed_precision_b200 import starkv as S
        self.S = S
        bf = lambda a: torch.from_numpy(gen.bf16_bits(a).view(np.int16).copy()).view(torch.bfloat16).to(device)
        f = gen.make_factors(w, seed)
        B, T0, C = w.batch, w.ctx, w.chunk
        self.total = T0 + C
        cfg = S.make_config(w.H, w.h_kv, w.d_h, w.hidden, w.r_k, w.R, self.total + 16, w.top_fraction, w.rope_base)
        self.kv = S.StarKV(cfg, bf(f.A_k), bf(f.A_v), bf(f.B_k), bf(f.B_v))
        bt, n_pages = gen.make_block_table(np.full(B, self.total, np.int32), seed)
        self.cache = self.kv.new_cache(n_pages)
        step = 4096
        for b in range(B):
            for s0 in range(0, T0, step):
                n = min(step, T0 - s0)
                X = bf(gen.make_hidden(n, w.hidden, seed, name="X", sub=1000 * b + s0 // step))
                slots = torch.from_numpy(gen.slots_for(bt, b, np.arange(s0, s0 + n))).to(device)
                self.kv.append(self.cache, X, slots)
        torch.cuda.synchronize()
        self.X = bf(gen.make_hidden(B * C, w.hidden, seed, name="X_chunk"))
        self.slots = torch.from_numpy(np.concatenate([gen.slots_for(bt, b, np.arange(T0, T0 + C))
                                                      for b in range(B)])).to(device)
        self.q = bf(gen.make_queries(B * C, w.H, w.d_h, seed, name="q_chunk"))
        self.cu_q = torch.tensor(np.arange(B + 1, dtype=np.int32) * C).to(device)
        self.bt = torch.from_numpy(bt).to(device)
        self.sl = torch.full((B,), self.total, dtype=torch.int32, device=device)
        self.out = torch.empty_like(self.q)
        self.ws = self.kv.workspace(S.OP_PREFILL, B, bt.shape[1], B * C)
        st = self.kv.status()
        if st:
            raise RuntimeError(f"device status {st:#x} after cache fill")

    def step(self, i=0, ev=None):
        S = self.S
        S.starkv_append(self.kv.ctx, self.cache.struct, self.X, self.slots)
        if ev is not None:
            ev[0].record()
        S.starkv_prefill_attn(self.kv.ctx, self.cache.struct, self.q, self.cu_q, self.bt, self.sl,
                              self.q.shape[0] // self.sl.shape[0], self.out, self.ws)
        if ev is not None:
            ev[1].record()


def prefill_flops(w) -> dict:
    """Algorithmic flops of one prefill step (causal QK and PV, values and keys
    re-expanded once per position and KV head, the chunk's projection)."""
    T0, C = w.ctx, w.chunk
    pairs = C * T0 + C * (C + 1) // 2                       # (query, key) pairs of one sequence
    attn = pairs * w.H * 4 * w.d_h
    vexp = (T0 + C) * w.h_kv * w.R * w.d_h * 2
    kexp = (T0 + C) * w.h_kv * w.r_k * w.d_h * 2
    proj = C * w.hidden * (w.h_kv * w.r_k + w.R) * 2
    per = {"attention": attn, "value_reexpansion": vexp, "key_reexpansion": kexp, "projection": proj}
    return {k: v * w.batch for k, v in per.items()}


PREFILL_DTYPE = "fp16 tensor-core operands, fp32 accumulation"
PREFILL_KERNELS = "tcgen05 key/value re-expansion + tcgen05 flash attention"


def prefill_launches_per_step(max_pages: int, n_append: int) -> int:
    """Kernels one prefill step launches: the append (the general kernel above
    64 tokens, else the split-K projection and the quantiser) and the prefill
    (re-expansion, then attention)."""
    return (1 if n_append > 64 else 2) + 2


# ---------------------------------------------------------------------------
# CPU oracle baselines (bounded samples, host cores; a baseline, not a target)
# ---------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def _timed(fn, seconds, at_least=1):
    done, t0 = 0, time.perf_counter()
    while True:
        fn()
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds and done >= at_least:
            return done, el


def _one_thread(fn, seconds):
    try:
        from threadpoolctl import threadpool_limits
    except Exception:
        return None
    with threadpool_limits(limits=1):
        return _timed(fn, seconds)


def _oracle_setup(w, seed, b, extra=0):
    import oracle as O
    cfg = O.config_of(w)
    L = int(gen.make_seq_lens(w, seed)[b])
    bt, n_pages = gen.make_block_table([L + extra], seed)
    oc = O.new_cache(cfg, n_pages)
    zk, zv = gen.make_latents(w, L, seed, sub=b)
    O.write_latents(oc, gen.slots_for(bt, 0, np.arange(L)), zk, zv)
    f = gen.make_factors(w, seed)
    q = gen.make_queries(1, w.H, w.d_h, seed, name="q_step", sub=b)
    return O, oc, bt, L, f, q


def cpu_baseline(w, seed, seconds):
    """One oracle decode call of one whole sequence (all heads), repeated for
    about `seconds`; then the same call on one BLAS thread."""
    O, oc, bt, L, f, q = _oracle_setup(w, seed, 0)
    call = lambda: O.decode(oc, q, f.B_k, f.B_v, bt, [L])
    done, el = _timed(call, seconds)
    rec = {"value": done * L / el, "unit": "context-tokens/s", "cores": _blas_threads(), "kind": "oracle",
           "sample": f"{done} oracle decode call(s) of one {L}-token sequence, all {w.H} heads, "
                     f"fp64 numpy, {el:.1f} s", "host_cpu_count": os.cpu_count()}
    one = _one_thread(call, seconds / 4)
    if one:
        rec["one_thread"] = {"value": one[0] * L / one[1], "cores": 1,
                             "sample": f"{one[0]} call(s) of the same sequence on one BLAS thread, {one[1]:.1f} s"}
    return rec


def cpu_baseline_stream(w, seed, n_steps=8):
    """The first n_steps stream steps on the oracle: append one token (projection,
    rotation, quantiser, packing) then decode the grown context, per step."""
    O, oc, bt, L0, f, _ = _oracle_setup(w, seed, 0, extra=n_steps)
    X = [gen.make_hidden(1, w.hidden, seed, name="X_step", sub=s) for s in range(n_steps)]
    q = [gen.make_queries(1, w.H, w.d_h, seed, name="q_step", sub=s) for s in range(n_steps)]
    state = {"s": 0}

    def step():
        s = state["s"]
        O.append(oc, X[s % n_steps], f.A_k, f.A_v, gen.slots_for(bt, 0, [L0 + s % n_steps]))
        O.decode(oc, q[s % n_steps], f.B_k, f.B_v, bt, [L0 + s % n_steps + 1])
        state["s"] += 1

    t0 = time.perf_counter()
    for _ in range(n_steps):
        step()
    el = time.perf_counter() - t0
    tokens = sum(L0 + s + 1 for s in range(n_steps))
    rec = {"value": tokens / el, "unit": "context-tokens/s", "cores": _blas_threads(), "kind": "oracle",
           "sample": f"the first {n_steps} stream steps (append 1 token + decode of {L0 + 1}..{L0 + n_steps} "
                     f"tokens, all {w.H} heads), fp64 numpy, {el:.1f} s, {el / n_steps:.2f} s per step",
           "seconds_per_step": el / n_steps, "host_cpu_count": os.cpu_count()}
    hs = list(range(max(1, w.H // 8)))
    one = _one_thread(lambda: O.decode(oc, q[0], f.B_k, f.B_v, bt, [L0 + 1], heads=hs), 0.0)
    if one:
        rec["one_thread"] = {"value": (L0 + 1) * (len(hs) / w.H) * one[0] / one[1], "cores": 1,
                             "sample": f"{one[0]} decode(s) of the first stream step's {L0 + 1} tokens on one "
                                       f"BLAS thread, {len(hs)} of {w.H} heads (counted as {len(hs)}/{w.H} of "
                                       f"its tokens), {one[1]:.1f} s"}
    return rec


def prefill_sample_flops(w, n_q: int, L: int) -> float:
    """Algorithmic flops of n_q queries at positions L - n_q .. L - 1 of one
    sequence: their causal attention pairs, plus their share (n_q of the chunk's
    queries) of one sequence's key/value re-expansion and projection."""
    fl = prefill_flops(w)
    pairs = sum(L - n_q + i + 1 for i in range(n_q))
    rest = (fl["value_reexpansion"] + fl["key_reexpansion"] + fl["projection"]) / w.batch
    return pairs * w.H * 4 * w.d_h + rest * n_q / w.chunk


def cpu_baseline_prefill(w, seed, seconds, n_q=4):
    O, oc, bt, L, f, _ = _oracle_setup(w, seed, 0)
    q = gen.make_queries(n_q, w.H, w.d_h, seed, name="q_chunk")
    call = lambda: O.prefill(oc, q, [0, n_q], f.B_k, f.B_v, bt, [L])
    done, el = _timed(call, seconds)
    fl = prefill_sample_flops(w, n_q, L)
    rec = {"value": done * fl / el / 1e12, "unit": "TFLOP/s",
           "cores": _blas_threads(), "kind": "oracle",
           "sample": f"{done} oracle prefill call(s) of {n_q} queries at the end of one {L}-token sequence, "
                     f"all {w.H} heads, fp64 numpy, {el:.1f} s", "host_cpu_count": os.cpu_count()}
    one = _one_thread(call, seconds / 4)
    if one:
        rec["one_thread"] = {"value": one[0] * fl / one[1] / 1e12, "cores": 1,
                             "sample": f"{one[0]} call(s) of the same sample on one BLAS thread, {one[1]:.1f} s"}
    return rec


# ---------------------------------------------------------------------------
# legs
# ---------------------------------------------------------------------------
def _timed_region(st, args, world, local, n_steps, timed_steps=None):
    """Warm-up, the timed steps (CUDA events on the launching stream, barriers
    on both sides) and a repeat pass of at least --sustain-seconds, all inside
    one clock sampler.  Returns (step ms total, per-step call events, sustained
    (n, ms/step), clocks of the timed region + repeat pass)."""
    import torch
    with ClockSampler(local) as clk:
        for i in range(args.warmup):
            st.step(i)
        torch.cuda.synchronize()
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(n_steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        clk.mark("timed")
        t0.record()
        for i in range(n_steps):
            st.step(i, pairs[i])
        t1.record()
        torch.cuda.synchronize()
        barrier(world)
        ms_step = t0.elapsed_time(t1) / max(1, n_steps)
        sus = sustained_pass(st.step, n_steps, args.sustain_seconds, ms_step) if args.sustain_seconds > 0 else None
        torch.cuda.synchronize()
        clk.mark("after")
    return t0.elapsed_time(t1), pairs, sus, clk.summary("timed", "after")


def run_prefill(args, w, rank, world, local, with_cpu=True, n_steps=None):
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    n_steps = n_steps or args.steps
    st = PrefillState(w, args.seed, device)
    ms, pairs, sus, clocks = _timed_region(st, args, world, local, n_steps)
    if st.kv.status():
        raise RuntimeError("device status set during the timed region")
    fl = prefill_flops(w)
    total = sum(fl.values())
    value, ms_max = job_throughput(total * n_steps / 1e12, ms, world, device)
    attn_ms = sum(a.elapsed_time(b) for a, b in pairs) / n_steps
    # ---- end to end through the public API with host buffers: the step's
    # inputs packed in one pinned staging buffer, one copy each way
    srcs = [st.X.cpu(), st.slots.cpu(), st.q.cpu(), st.cu_q.cpu(), st.bt.cpu(), st.sl.cpu()]
    offs, h2d = pack_layout(srcs)
    hbuf = torch.zeros(h2d, dtype=torch.uint8).pin_memory()
    for v, x in zip(packed_views(hbuf, offs, srcs), srcs):
        v.copy_(x)
    dbuf = torch.empty(h2d, dtype=torch.uint8, device=device)
    Xd, sld, qd, cud, btd, lnd = packed_views(dbuf, offs, srcs)
    outh = torch.empty(st.out.shape, dtype=torch.bfloat16).pin_memory()
    d2h = outh.numel() * outh.element_size()
    S = st.S

    def e2e_step():
        dbuf.copy_(hbuf, non_blocking=True)
        S.starkv_append(st.kv.ctx, st.cache.struct, Xd, sld)
        S.starkv_prefill_attn(st.kv.ctx, st.cache.struct, qd, cud, btd, lnd, w.chunk, st.out, st.ws)
        outh.copy_(st.out, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    e2e_value, _ = job_throughput(total * n_steps / 1e12, e0.elapsed_time(e1), world, device)
    if rank != 0:
        return None
    peak, peak_kind = measured_tensor_peak()
    achieved = (total - fl["projection"]) / (attn_ms / 1e3) / 1e12
    traffic, tnote = dram_traffic(w.name, "prefill_call")
    line = {
        "metric": "prefill TFLOP/s (algorithmic)", "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": n_steps, "warmup": args.warmup, "ms_per_step": ms_max / n_steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": PREFILL_DTYPE, "data": "synthetic (seeded)",
        "config": {"workload": w.name, "batch": w.batch, "ctx": w.ctx, "chunk": w.chunk,
                   "step": "append the chunk + causal prefill attention of its queries",
                   "l2": f"cache {st.cache.nbytes() / 2**20:.0f} MiB read per step (vs 126 MiB L2)"},
        "flops_per_step": fl,
        "roofline": {"bound": "tensor", "kernel": "starkv_prefill_attn (" + PREFILL_KERNELS + ")",
                     "achieved": achieved, "peak": peak, "peak_kind": f"bf16 dense TFLOP/s ({peak_kind}); "
                     "fp16 operands share the nominal dense rate", "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": traffic, "traffic_source": tnote, "launch_ms": attn_ms},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": prefill_launches_per_step(int(st.bt.shape[1]), w.batch * w.chunk) * n_steps,
        "clocks": clocks,
    }
    if sus:
        line["sustained"] = sustained_record(sus[0], sus[1], total / 1e12, clocks, "TFLOP/s")
    if world == 1 and with_cpu:
        line["cpu_baseline"] = cpu_baseline_prefill(w, args.seed, args.cpu_seconds)
    return line


def decode_launches_per_step(n_append: int) -> int:
    """Kernels of one decode step: the append (split-K projection + quantiser for
    up to 64 tokens, one fused kernel above) and the decode (query fold, scores,
    values, projection)."""
    return (2 if n_append <= 64 else 1) + 4


def _decode_line(w, args, world, st, n_steps, ms_max, dec_ms, value, tokens_per_step, e2e, clocks, sus, cfg_extra):
    peak, peak_kind = measured_peaks()
    alg = decode_algorithmic_bytes(w, tokens_per_step, w.batch, st.max_pages)
    achieved = alg / (dec_ms / 1e3) / 1e9
    traffic, tnote = dram_traffic(w.name, "decode_call")
    line = {
        "metric": "decode context-tokens/s",
        "value": value,
        "unit": "context-tokens/s",
        "n_gpus": world,
        "steps": n_steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max / n_steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp16 tensor-core operands, fp32 accumulation",
        "data": "synthetic (seeded; shapes of the named model, no weights)",
        "config": {"workload": w.name, "batch": w.batch,
                   "heads": w.H, "kv_heads": w.h_kv, "head_dim": w.d_h, "rank_k": w.r_k, "rank_v": w.R,
                   "bits": "4/3 (top 25% of channels 4-bit)", "page_tokens": 16,
                   "parallelism": f"dp{world} (independent sequences per GPU)",
                   "l2": f"{len(st.caches)} rotating cache replicas "
                         f"({len(st.caches) * st.caches[0].nbytes() / 2**20:.0f} MiB > 126 MiB L2)", **cfg_extra},
        "roofline": {"bound": "hbm", "kernel": "starkv_decode_attn (query fold + scores + values + projection)",
                     "achieved": achieved, "peak": peak, "peak_kind": f"hbm copy GB/s ({peak_kind})",
                     "unit": "GB/s", "frac": achieved / peak, "spec_gbs": SPEC_HBM_GBS,
                     "frac_of_spec": achieved / SPEC_HBM_GBS, "traffic": traffic, "traffic_source": tnote,
                     "algorithmic_bytes_per_launch": alg, "launch_ms": dec_ms,
                     "achieved_context_tokens_per_s_decode_only": tokens_per_step / (dec_ms / 1e3)},
        "e2e": e2e,
        "gpu_launches": decode_launches_per_step(w.batch) * n_steps,
        "clocks": clocks,
    }
    if sus:
        line["sustained"] = sustained_record(sus[0], sus[1], tokens_per_step, clocks, "context-tokens/s")
    return line


def run_starkv(args, w, rank, world, local, with_cpu=True, n_steps=None):
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    n_steps = n_steps or args.steps
    replicas = max(1, int(np.ceil(3 * L2_BYTES / max(1, w.batch * w.ctx * bytes_per_token(w)))))
    replicas = max(replicas, 2)
    st = DecodeState(w, args.seed, device, replicas)
    S = st.S
    ms, pairs, sus, clocks = _timed_region(st, args, world, local, n_steps)
    dec_ms = sum(a.elapsed_time(b) for a, b in pairs) / n_steps
    status = st.kv.status()
    if status:
        raise RuntimeError(f"device status {status:#x} during the timed region")
    tokens_per_step = int(st.seq_lens.sum())
    value, ms_max = job_throughput(tokens_per_step * n_steps, ms, world, device)
    # ---- end to end through the public API with host buffers: the step's
    # inputs sit packed in one pinned staging buffer and cross in one copy
    t_ = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    srcs = [t_(gen.bf16_bits(st.X_np).view(np.int16)).view(torch.bfloat16),
            t_(gen.bf16_bits(st.q_np).view(np.int16)).view(torch.bfloat16),
            t_(st.slots_np), t_(st.bt_np), t_(st.seq_lens.astype(np.int32))]
    offs, h2d = pack_layout(srcs)
    hbuf = torch.zeros(h2d, dtype=torch.uint8).pin_memory()
    for v, s in zip(packed_views(hbuf, offs, srcs), srcs):
        v.copy_(s)
    dbuf = torch.empty(h2d, dtype=torch.uint8, device=device)
    Xd, qd, sld, btd, ld = packed_views(dbuf, offs, srcs)
    outh = torch.empty(st.q.shape, dtype=torch.bfloat16).pin_memory()
    d2h = outh.numel() * outh.element_size()

    def e2e_step(i):
        dbuf.copy_(hbuf, non_blocking=True)
        c = st.caches[i % len(st.caches)]
        S.starkv_append(st.kv.ctx, c.struct, Xd, sld)
        S.starkv_decode_attn(st.kv.ctx, c.struct, qd, btd, ld, st.out, st.ws)
        outh.copy_(st.out, non_blocking=True)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n_steps):
        e2e_step(i)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    e2e_value, _ = job_throughput(tokens_per_step * n_steps, e0.elapsed_time(e1), world, device)

    if rank != 0:
        return None
    e2e = {"value": e2e_value, "unit": "context-tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    extra = {"ctx": int(st.seq_lens.max()), "ctx_min": int(st.seq_lens.min()),
             "step": "append 1 token per sequence + decode attention"}
    line = _decode_line(w, args, world, st, n_steps, ms_max, dec_ms, value, tokens_per_step, e2e, clocks, sus, extra)
    if world == 1 and with_cpu:
        line["cpu_baseline"] = cpu_baseline(w, args.seed, args.cpu_seconds)
    return line


def run_stream(args, w, rank, world, local, with_cpu=True, n_steps=None):
    """Long-context stream: each timed step appends one token per sequence and
    decodes the grown context; the run walks the stream's steps in order."""
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    n_steps = n_steps or args.steps
    replicas = max(2, int(np.ceil(3 * L2_BYTES / max(1, w.batch * w.ctx * bytes_per_token(w)))))
    st = StreamState(w, args.seed, device, replicas)
    S = st.S
    ms, pairs, sus, clocks = _timed_region(st, args, world, local, n_steps)
    dec_ms = sum(a.elapsed_time(b) for a, b in pairs) / n_steps
    status = st.kv.status()
    if status:
        raise RuntimeError(f"device status {status:#x} during the timed region")
    tokens = sum(st.tokens(i) for i in range(n_steps))
    value, ms_max = job_throughput(tokens, ms, world, device)
    # ---- end to end through the public API with host buffers: each stream
    # step's inputs sit packed in one row of a pinned staging buffer
    t_ = lambda a: torch.from_numpy(np.ascontiguousarray(a))

    def host_inputs(s):
        return [t_(gen.bf16_bits(st.X_np[s]).view(np.int16)).view(torch.bfloat16),
                t_(gen.bf16_bits(st.q_np[s]).view(np.int16)).view(torch.bfloat16),
                t_(st.slots_np[s]), t_(st.bt_np), t_(st.lens_np[s])]

    offs, h2d = pack_layout(host_inputs(0))
    pitch = -(-h2d // 256) * 256  # rows start aligned for every view's dtype
    hbuf = torch.zeros((st.n, pitch), dtype=torch.uint8).pin_memory()
    for s in range(st.n):
        srcs = host_inputs(s)
        for v, x in zip(packed_views(hbuf[s], offs, srcs), srcs):
            v.copy_(x)
    dbuf = torch.empty(h2d, dtype=torch.uint8, device=device)
    Xd, qd, sld, btd, ld = packed_views(dbuf, offs, host_inputs(0))
    outh = torch.empty(st.out.shape, dtype=torch.bfloat16).pin_memory()
    d2h = outh.numel() * outh.element_size()

    def e2e_step(i):
        dbuf.copy_(hbuf[i % st.n, :h2d], non_blocking=True)
        c = st.caches[i % len(st.caches)]
        S.starkv_append(st.kv.ctx, c.struct, Xd, sld)
        S.starkv_decode_attn(st.kv.ctx, c.struct, qd, btd, ld, st.out, st.ws)
        outh.copy_(st.out, non_blocking=True)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n_steps):
        e2e_step(i)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    e2e_value, _ = job_throughput(tokens, e0.elapsed_time(e1), world, device)

    if rank != 0:
        return None
    mean_tokens = tokens / n_steps
    L0, Ln = int(st.L0.max()), int(st.L0.max()) + st.n
    e2e = {"value": e2e_value, "unit": "context-tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    extra = {"ctx": f"{L0} -> {Ln}",
             "step": f"append 1 token per sequence + decode of the grown context; "
                     f"run step i is stream step i mod {st.n}"}
    line = _decode_line(w, args, world, st, n_steps, ms_max, dec_ms, value, mean_tokens, e2e, clocks, sus, extra)
    if world == 1 and with_cpu:
        line["cpu_baseline"] = cpu_baseline_stream(w, args.seed)
    return line


def run_reference(args, w, rank, world):
    """The fp64 CPU oracle on the same workload; each step is a bounded sample:
    one sequence of the batch and a subset of its heads, sized so the whole run
    stays within a few minutes."""
    if rank != 0:
        return None
    if w.chunk > 0:
        return _run_reference_prefill(args, w, world)
    O, oc, bt, L, f, q = _oracle_setup(w, args.seed, 0)
    t0 = time.perf_counter()
    O.decode(oc, q, f.B_k, f.B_v, bt, [L])
    t_full = time.perf_counter() - t0
    cap_s = 150.0  # host seconds the timed oracle steps may take
    heads = max(1, min(w.H, int(w.H * cap_s / max(1e-9, args.steps * t_full))))
    hs = list(range(heads))
    for _ in range(min(args.warmup, 1)):
        O.decode(oc, q, f.B_k, f.B_v, bt, [L], heads=hs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.decode(oc, q, f.B_k, f.B_v, bt, [L], heads=hs)
    el = time.perf_counter() - t0
    v = args.steps * L * (heads / w.H) / el
    sample = f"each step: one {L}-token sequence, {heads} of {w.H} heads (counted as {heads}/{w.H} of its tokens)"
    return {
        "metric": "decode context-tokens/s", "value": v, "unit": "context-tokens/s", "impl": "reference",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": w.name, "batch": w.batch, "ctx": w.ctx, "sample": sample},
        "cpu_baseline": {"value": v, "unit": "context-tokens/s", "cores": _blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": "context-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def _run_reference_prefill(args, w, world, n_q=4):
    """Prefill workloads: each step is n_q queries at the end of one sequence,
    on a subset of the heads sized so the run stays within a few minutes;
    flops are the sample's algorithmic share, scaled by the heads taken."""
    O, oc, bt, L, f, _ = _oracle_setup(w, args.seed, 0)
    q = gen.make_queries(n_q, w.H, w.d_h, args.seed, name="q_chunk")
    t0 = time.perf_counter()
    O.prefill(oc, q, [0, n_q], f.B_k, f.B_v, bt, [L])
    t_full = time.perf_counter() - t0
    heads = max(1, min(w.H, int(w.H * 150.0 / max(1e-9, args.steps * t_full))))
    hs = list(range(heads))
    for _ in range(min(args.warmup, 1)):
        O.prefill(oc, q, [0, n_q], f.B_k, f.B_v, bt, [L], heads=hs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.prefill(oc, q, [0, n_q], f.B_k, f.B_v, bt, [L], heads=hs)
    el = time.perf_counter() - t0
    v = args.steps * prefill_sample_flops(w, n_q, L) * (heads / w.H) / el / 1e12
    sample = (f"each step: {n_q} queries at the end of one {L}-token sequence, {heads} of {w.H} heads "
              f"(counted as {heads}/{w.H} of their algorithmic flops)")
    return {
        "metric": "prefill TFLOP/s (algorithmic)", "value": v, "unit": "TFLOP/s", "impl": "reference",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": w.name, "batch": w.batch, "ctx": w.ctx, "chunk": w.chunk, "sample": sample},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_leg(args, w, rank, world, local, with_cpu, n_steps=None):
    if w.chunk > 0:
        return run_prefill(args, w, rank, world, local, with_cpu, n_steps)
    if w.steps > 0:
        return run_stream(args, w, rank, world, local, with_cpu, n_steps)
    return run_starkv(args, w, rank, world, local, with_cpu, n_steps)


def subrecord_steps(w, steps: int) -> int:
    """Timed steps of a workload's record: the stream walks all its steps at least once;
    a prefill step is a long call, so at most 10 are timed."""
    if w.steps > 0:
        return max(steps, w.steps)
    if w.chunk > 0:
        return max(1, min(steps, 10))
    return steps


def main(argv=None):
    argv = list(sys.argv[1:] if argv is None else argv)
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="starkv", choices=["starkv", "reference"])
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--only", action="store_true", help="the named workload alone, without the other records")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--sustain-seconds", type=float, default=1.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "starkv":
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        rc = launch_ranks(args.gpus, argv)
        if rc:
            raise SystemExit(rc)
        return
    rank, world, local = dist_env()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but {world} ranks were launched")
    w = gen.workload(args.workload)
    if args.impl == "reference":
        line = run_reference(args, w, rank, world)
    else:
        line = run_leg(args, w, rank, world, local, not args.no_cpu_baseline)
        if world == 1 and not args.only and line is not None:
            recs = {}
            for name in SUBRECORDS:
                if name == w.name:
                    continue
                ws = gen.workload(name)
                recs[name] = run_leg(args, ws, rank, world, local, not args.no_cpu_baseline,
                                     subrecord_steps(ws, args.steps))
            if recs:
                line["workloads"] = recs
    if line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
