"""Sequence (context) sharding of decode across GPUs.

One long sequence's context is split into contiguous slices, one per rank;
each rank holds its slice's packed latents in its own cache.  A decode step
then runs ``starkv_decode_attn_slice`` on every rank (its keys RoPE'd at their
global positions, the query at the sequence's last position), exchanges the
per-slice results, (o, m, l) with o d_h wide after the B_v projection (B_v is
linear, so each slice projects locally), with one all-gather, and merges them
with ``starkv_merge_slices``: the softmax partition identity (attention
decomposition theorem, eq. 1 of the CaliDrop review) makes the merge exact.

This module is plumbing only: the slice attention and the merge run in the
CUDA library; the exchange is ``torch.distributed`` (NCCL over NVLink on GPUs).
"""
from __future__ import annotations

import torch

from . import starkv as S


def token_ranges(n_tokens: int, world: int):
    """Contiguous, balanced slices [lo, hi) of n_tokens positions, one per rank
    (earlier ranks take the remainder)."""
    if world < 1 or n_tokens < 0:
        raise ValueError("world must be >= 1 and n_tokens >= 0")
    base, extra = divmod(n_tokens, world)
    out, lo = [], 0
    for r in range(world):
        hi = lo + base + (1 if r < extra else 0)
        out.append((lo, hi))
        lo = hi
    return out


def slice_of(n_tokens: int, rank: int, world: int):
    return token_ranges(n_tokens, world)[rank]


class SlicePlan:
    """Per-rank arguments of a sharded decode step: the local token counts, the
    global position of each local slice's first token, and the query position."""

    def __init__(self, total_lens, rank: int, world: int, device):
        lo_hi = [slice_of(int(n), rank, world) for n in total_lens]
        self.local_lens = torch.tensor([hi - lo for lo, hi in lo_hi], dtype=torch.int32, device=device)
        self.key_pos0 = torch.tensor([lo for lo, _ in lo_hi], dtype=torch.int32, device=device)
        self.q_pos = torch.tensor([max(int(n) - 1, 0) for n in total_lens], dtype=torch.int32, device=device)
        self.ranges = lo_hi


def gather_slices(o, ml, group=None):
    """All-gather the per-rank slice results: returns [world, ...] stacks."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    o_all = [torch.empty_like(o) for _ in range(world)]
    ml_all = [torch.empty_like(ml) for _ in range(world)]
    dist.all_gather(o_all, o, group=group)
    dist.all_gather(ml_all, ml, group=group)
    return torch.stack(o_all), torch.stack(ml_all)


def decode_sharded(kv, cache, q, block_table, plan: SlicePlan, workspace, out=None, group=None, stream=None):
    """One sharded decode step on this rank: slice attention, all-gather, merge.

    kv: the rank's StarKV context; cache: its LatentCache (the local slices);
    block_table: the local pages of each sequence's slice; q: [B, H, d] bf16
    (the same queries on every rank).  Returns the bf16 output [B, H, d]."""
    B, H, d = q.shape
    o = torch.empty((B, H, d), dtype=torch.float32, device=q.device)
    ml = torch.empty((B, H, 2), dtype=torch.float32, device=q.device)
    S.starkv_decode_attn_slice(kv.ctx, cache.struct, q, block_table, plan.local_lens, plan.key_pos0, plan.q_pos,
                               o, ml, workspace, stream)
    o_all, ml_all = gather_slices(o, ml, group)
    if out is None:
        out = torch.empty_like(q)
    S.starkv_merge_slices(kv.ctx, o_all.contiguous(), ml_all.contiguous(), out, stream)
    return out
