"""Data parallelism for the LoRA layer: shard the tokens (M), sum the adapter
gradients.

The layer is row-wise in X, so data parallelism along M needs no exchange in
the forward and only one in the backward: every rank computes dX for its own
rows and partial dA, dB over its own rows; the full-batch gradients are the
sums of the partials over ranks (dA = sum_g dT_g^T X_g, dB = s sum_g dY_g^T T_g).
W is frozen and every rank merges its own replica, so the merge has no
exchange either.  (fastaf 0.1.0, "Contributing & Roadmap": the kernels assume
the full weight on each device; tensor parallelism is not supported.)

Only torch.distributed is used here (NCCL on GPUs, gloo on CPUs).
"""
from __future__ import annotations

from typing import Tuple


def shard_rows(M: int, world: int, rank: int) -> Tuple[int, int]:
    """[begin, end) of this rank's rows when M tokens are split as evenly as
    possible over `world` ranks (the first M % world ranks get one more)."""
    if world <= 0 or not (0 <= rank < world):
        raise ValueError(f"bad rank {rank} of {world}")
    base, extra = divmod(int(M), int(world))
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def allreduce_adapter_grads(dA, dB, group=None, async_op: bool = False):
    """Sum dA and dB over the ranks of `group`, in place (one all-reduce
    each; the same collective order on every rank).  With async_op the two
    collectives are only enqueued (on NCCL they start once the work already
    on the current stream is done) and their work handles are returned, so
    that later kernels (the dX step) run while they are in flight; call
    .wait() on each before dA and dB are read."""
    import torch.distributed as dist
    w1 = dist.all_reduce(dA, op=dist.ReduceOp.SUM, group=group, async_op=async_op)
    w2 = dist.all_reduce(dB, op=dist.ReduceOp.SUM, group=group, async_op=async_op)
    return [w1, w2] if async_op else None


def max_over_ranks(values, device=None, group=None):
    """Element-wise maximum of a list of floats over the ranks (timing)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return [float(v) for v in t.tolist()]
