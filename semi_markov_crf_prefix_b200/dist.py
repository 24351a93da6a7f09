"""Data-parallel helpers: sequences are independent, so a batch shards across
ranks by sequence and the only exchange is the sum of the shared-parameter
gradients dA [C, C] and dD [K, C] (float64) over ranks.  log Z and dX stay on the
rank that owns the sequence.  The recursion is sequential along T, so a single
sequence is never split.

These are host-side helpers over torch.distributed (NCCL on GPUs, gloo on CPU);
they hold none of the semi-CRF arithmetic.
"""
from __future__ import annotations


def shard_range(B: int, world: int, rank: int):
    """Contiguous block of sequence indices [lo, hi) owned by `rank`.

    Blocks differ in size by at most one; ranks beyond B get an empty range.
    """
    if world < 1 or not (0 <= rank < world):
        raise ValueError("need 0 <= rank < world")
    base, extra = divmod(B, world)
    lo = rank * base + min(rank, extra)
    hi = lo + base + (1 if rank < extra else 0)
    return lo, hi


def reduce_param_grads(dA, dD, group=None):
    """Sum dA and dD over all ranks in place (one all-reduce, both tensors).

    The two gradients are packed into one contiguous buffer so the exchange is
    a single collective (C*C + K*C float64 values).
    """
    import torch
    import torch.distributed as dist
    flat = torch.cat([dA.reshape(-1), dD.reshape(-1)])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    dA.copy_(flat[: dA.numel()].view_as(dA))
    dD.copy_(flat[dA.numel():].view_as(dD))
    return dA, dD
