"""Data-parallel plumbing for the scan path (one process per GPU).

Batch elements are independent (B and C are per batch element), so the path
shards by batch with no exchange inside the scan; the only cross-rank step in
data-parallel training is the sum of the per-channel parameter gradients
(dD, dconv_w, dconv_b), which belongs to the caller's training step.  These
helpers take any torch.distributed process group (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

PARAM_GRADS = ("dD", "dconv_w", "dconv_b")


def shard_batch(global_batch: int, rank: int, world: int) -> tuple[int, int]:
    """[start, stop) of this rank's batch elements: contiguous, disjoint,
    covering the batch, sizes differing by at most one."""
    if global_batch < 0 or world < 1 or not 0 <= rank < world:
        raise ValueError("bad shard arguments")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_param_grads(grads: dict, group=None) -> dict:
    """Sum the per-channel parameter gradients over ranks, in place."""
    for k in PARAM_GRADS:
        g = grads.get(k)
        if g is not None:
            dist.all_reduce(g, op=dist.ReduceOp.SUM, group=group)
    return grads


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The largest `value` over ranks (timings: the job is as slow as its
    slowest rank)."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
