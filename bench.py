"""Benchmark: decode context-tokens/s and achieved HBM GB/s of STAR-KV latent-cache attention.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl starkv|reference] [--workload NAME]

One step = one pass of the decode hot path over one batch: append one new token
per sequence (project, rotate, quantise, pack) and then batched single-query
attention over the packed cache (dequantise, re-expand and RoPE keys, online
softmax, P Z_v in the latent, split merge, B_v projection).  Default workload:
LongChat-7B-shaped layer, 32 heads, d_h 128, r_k 32, R 1024, batch 16, context
4096, 16-token pages.  Inputs are seeded and synthetic (no weights or datasets).

For N > 1 (torchrun), every rank runs its own batch of independent sequences
(weak scaling, no collective on the data path); the timing is the maximum over
ranks.  The reference arm times the fp64 CPU oracle on a bounded sample of the
same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from harness import gen  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0

# DRAM bytes (read + write) of one decode call, summed over its four kernels,
# from one ncu capture of the current kernels (profiles/decode_kernels_*.md);
# None for a workload without a capture.  Reset whenever a decode kernel changes.
DECODE_TRAFFIC_NCU: dict = {}
# The last capture, taken before the projection kernel's loads were reordered
# (same loads and bytes, issued earlier); reported under its own key, never as
# `traffic`.
DECODE_TRAFFIC_LAST_CAPTURE = {"longchat7b_decode_b16_t4096": 134_520_000}


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


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            p = [x.strip() for x in l.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx.append(float(p[2]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


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

    def step(self, ev=None):
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


def prefill_launches_per_step(max_pages: int, n_append: int) -> int:
    """Kernels one prefill step launches: the append (the general kernel above
    64 tokens, else the split-K projection and the quantiser) and the prefill
    (init, then expand + attention per key chunk of up to 512 positions, finalize)."""
    max_len = max_pages * 16
    chunk = 512 if max_len >= 512 else max(32, -(-max_len // 32) * 32)
    return (1 if n_append > 64 else 2) + 2 + 2 * (-(-max_len // chunk))


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
    done, t0 = 0, time.perf_counter()
    while True:
        O.prefill(oc, q, [0, n_q], f.B_k, f.B_v, bt, [L])
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": done * prefill_sample_flops(w, n_q, L) / el / 1e12, "unit": "TFLOP/s",
            "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{done} oracle prefill call(s) of {n_q} queries at the end of one {L}-token sequence, "
                      f"all {w.H} heads, fp64 numpy, {el:.1f} s", "host_cpu_count": os.cpu_count()}


def run_prefill(args, w, rank, world, local):
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    st = PrefillState(w, args.seed, device)
    for _ in range(args.warmup):
        st.step()
    torch.cuda.synchronize()
    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0.record()
        for i in range(args.steps):
            st.step(pairs[i])
        t1.record()
        torch.cuda.synchronize()
    barrier(world)
    if st.kv.status():
        raise RuntimeError("device status set during the timed region")
    fl = prefill_flops(w)
    total = sum(fl.values())
    value, ms_max = job_throughput(total * args.steps / 1e12, t0.elapsed_time(t1), world, device)
    attn_ms = sum(a.elapsed_time(b) for a, b in pairs) / args.steps
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
    for _ in range(args.steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    e2e_value, _ = job_throughput(total * args.steps / 1e12, e0.elapsed_time(e1), world, device)
    if rank != 0:
        return None
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        pass
    peak = float(peaks.get("bf16_tflops", 1590.0))
    achieved = (total - fl["projection"]) / (attn_ms / 1e3) / 1e12
    line = {
        "metric": "prefill TFLOP/s (algorithmic)", "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32 (CUDA-core prefill)", "data": "synthetic (seeded)",
        "config": {"workload": w.name, "batch": w.batch, "ctx": w.ctx, "chunk": w.chunk,
                   "step": "append the chunk + causal prefill attention of its queries",
                   "l2": f"cache {st.cache.nbytes() / 2**20:.0f} MiB read per step (vs 126 MiB L2)"},
        "flops_per_step": fl,
        "roofline": {"bound": "tensor", "kernel": "starkv_prefill_attn (expand + attention kernels)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": None, "launch_ms": attn_ms},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": prefill_launches_per_step(int(st.bt.shape[1]), w.batch * w.chunk) * args.steps,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_prefill(w, args.seed, args.cpu_seconds)
    return line


def run_starkv(args, w, rank, world, local):
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    replicas = max(1, int(np.ceil(3 * L2_BYTES / max(1, w.batch * w.ctx * bytes_per_token(w)))))
    replicas = max(replicas, 2)
    st = DecodeState(w, args.seed, device, replicas)
    S = st.S
    launches_per_step = 6  # append (split-K projection, quantise), decode (query fold, scores, values, projection)
    for i in range(args.warmup):
        st.step(i)
    torch.cuda.synchronize()
    # ---- device-resident timed region
    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0.record()
        for i in range(args.steps):
            st.step(i, pairs[i])
        t1.record()
        torch.cuda.synchronize()
    barrier(world)
    ms = t0.elapsed_time(t1)
    dec_ms = sum(a.elapsed_time(b) for a, b in pairs) / args.steps
    status = st.kv.status()
    if status:
        raise RuntimeError(f"device status {status:#x} during the timed region")
    tokens_per_step = int(st.seq_lens.sum())
    value, ms_max = job_throughput(tokens_per_step * args.steps, ms, world, device)
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
    for i in range(args.steps):
        e2e_step(i)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    e2e_value, _ = job_throughput(tokens_per_step * args.steps, e0.elapsed_time(e1), world, device)

    if rank != 0:
        return None
    peak, peak_kind = measured_peaks()
    alg = decode_algorithmic_bytes(w, tokens_per_step, w.batch, st.max_pages)
    achieved = alg / (dec_ms / 1e3) / 1e9
    line = {
        "metric": "decode context-tokens/s",
        "value": value,
        "unit": "context-tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp16 tensor-core operands, fp32 accumulation",
        "data": "synthetic (seeded; shapes of the named model, no weights)",
        "config": {"workload": w.name, "batch": w.batch, "ctx": int(st.seq_lens.max()),
                   "heads": w.H, "kv_heads": w.h_kv, "head_dim": w.d_h, "rank_k": w.r_k, "rank_v": w.R,
                   "bits": "4/3 (top 25% of channels 4-bit)", "page_tokens": 16,
                   "step": "append 1 token per sequence + decode attention",
                   "parallelism": f"dp{world} (independent sequences per GPU)",
                   "l2": f"{len(st.caches)} rotating cache replicas "
                         f"({len(st.caches) * st.caches[0].nbytes() / 2**20:.0f} MiB > 126 MiB L2)"},
        "roofline": {"bound": "hbm", "kernel": "starkv_decode_attn (scores + values + projection kernels)",
                     "achieved": achieved, "peak": peak, "peak_kind": f"hbm copy GB/s ({peak_kind})",
                     "unit": "GB/s", "frac": achieved / peak, "traffic": DECODE_TRAFFIC_NCU.get(w.name),
                     "traffic_last_capture": DECODE_TRAFFIC_LAST_CAPTURE.get(w.name),
                     "algorithmic_bytes_per_launch": alg, "launch_ms": dec_ms,
                     "achieved_context_tokens_per_s_decode_only": tokens_per_step / (dec_ms / 1e3)},
        "e2e": {"value": e2e_value, "unit": "context-tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.seed, args.cpu_seconds)
    return line


def run_stream(args, w, rank, world, local):
    """Long-context stream: each timed step appends one token per sequence and
    decodes the grown context; the run walks the stream's steps in order."""
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    replicas = max(2, int(np.ceil(3 * L2_BYTES / max(1, w.batch * w.ctx * bytes_per_token(w)))))
    st = StreamState(w, args.seed, device, replicas)
    S = st.S
    launches_per_step = 6  # append (split-K projection, quantise), decode (query fold, scores, values, projection)
    for i in range(args.warmup):
        st.step(i)
    torch.cuda.synchronize()
    # ---- device-resident timed region: stream steps 0, 1, ... in order
    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0.record()
        for i in range(args.steps):
            st.step(i, pairs[i])
        t1.record()
        torch.cuda.synchronize()
    barrier(world)
    ms = t0.elapsed_time(t1)
    dec_ms = sum(a.elapsed_time(b) for a, b in pairs) / args.steps
    status = st.kv.status()
    if status:
        raise RuntimeError(f"device status {status:#x} during the timed region")
    tokens = sum(st.tokens(i) for i in range(args.steps))
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
    for i in range(args.steps):
        e2e_step(i)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    e2e_value, _ = job_throughput(tokens, e0.elapsed_time(e1), world, device)

    if rank != 0:
        return None
    peak, peak_kind = measured_peaks()
    mean_tokens = tokens / args.steps
    alg = decode_algorithmic_bytes(w, mean_tokens, w.batch, st.max_pages)
    achieved = alg / (dec_ms / 1e3) / 1e9
    L0, Ln = int(st.L0.max()), int(st.L0.max()) + st.n
    line = {
        "metric": "decode context-tokens/s",
        "value": value,
        "unit": "context-tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp16 tensor-core operands, fp32 accumulation",
        "data": "synthetic (seeded; shapes of the named model, no weights)",
        "config": {"workload": w.name, "batch": w.batch, "ctx": f"{L0} -> {Ln}",
                   "heads": w.H, "kv_heads": w.h_kv, "head_dim": w.d_h, "rank_k": w.r_k, "rank_v": w.R,
                   "bits": "4/3 (top 25% of channels 4-bit)", "page_tokens": 16,
                   "step": f"append 1 token per sequence + decode of the grown context; "
                           f"run step i is stream step i mod {st.n}",
                   "parallelism": f"dp{world} (independent sequences per GPU)",
                   "l2": f"{len(st.caches)} rotating cache replicas "
                         f"({len(st.caches) * st.caches[0].nbytes() / 2**20:.0f} MiB > 126 MiB L2)"},
        "roofline": {"bound": "hbm", "kernel": "starkv_decode_attn (scores + values + projection kernels)",
                     "achieved": achieved, "peak": peak, "peak_kind": f"hbm copy GB/s ({peak_kind})",
                     "unit": "GB/s", "frac": achieved / peak, "traffic": DECODE_TRAFFIC_NCU.get(w.name),
                     "algorithmic_bytes_per_launch": alg, "launch_ms": dec_ms,
                     "achieved_context_tokens_per_s_decode_only": mean_tokens / (dec_ms / 1e3)},
        "e2e": {"value": e2e_value, "unit": "context-tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.seed, args.cpu_seconds)
    return line


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------
def _oracle_setup(w, seed, b):
    import oracle as O
    cfg = O.config_of(w)
    L = int(gen.make_seq_lens(w, seed)[b])
    bt, n_pages = gen.make_block_table([L], seed)
    oc = O.new_cache(cfg, n_pages)
    zk, zv = gen.make_latents(w, L, seed, sub=b)
    O.write_latents(oc, gen.slots_for(bt, 0, np.arange(L)), zk, zv)
    f = gen.make_factors(w, seed)
    q = gen.make_queries(1, w.H, w.d_h, seed, name="q_step", sub=b)
    return O, oc, bt, L, f, q


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def cpu_baseline(w, seed, seconds):
    O, oc, bt, L, f, q = _oracle_setup(w, seed, 0)
    done, t0 = 0, time.perf_counter()
    while True:
        O.decode(oc, q, f.B_k, f.B_v, bt, [L])
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": done * L / el, "unit": "context-tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{done} oracle decode call(s) of one {L}-token sequence, all {w.H} heads, "
                      f"fp64 numpy, {el:.1f} s", "host_cpu_count": os.cpu_count()}


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


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="starkv", choices=["starkv", "reference"])
    ap.add_argument("--workload", default="longchat7b_decode_b16_t4096")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "starkv":
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_env()
    w = gen.workload(args.workload)
    if args.impl == "reference":
        line = run_reference(args, w, rank, world)
    elif w.chunk > 0:
        line = run_prefill(args, w, rank, world, local)
    elif w.steps > 0:
        line = run_stream(args, w, rank, world, local)
    else:
        line = run_starkv(args, w, rank, world, local)
    if line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
