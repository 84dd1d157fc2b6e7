"""Multi-GPU plumbing for the transform: one process per GPU over torch.distributed.

The transform is token-parallel: every (token, head) row is independent given the RoPE
table and the pair angles, so ranks shard tokens with no collective on the data path.
The one real exchange is calibration: the pooled estimator adds the raw Q/K moment
accumulators of every calibration token ("When Local Variance Optimality Is Not
Enough ...", "Estimation strategies": raw accumulators pooled across heads before
centring), so the [2][d_h/2][6] fp64 accumulators are summed across ranks before the
closed-form solve, and every rank then solves the same angles.

These helpers work on any backend: NCCL with CUDA tensors on the GPU machine, gloo with
CPU tensors in the host-side tests.
"""
from __future__ import annotations

__all__ = ["token_shard", "pool_moments", "max_over_ranks"]


def token_shard(T: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous token range [start, stop) of ``rank`` when T tokens are split over
    ``world`` ranks (the first T % world ranks get one more token)."""
    if world < 1 or not 0 <= rank < world or T < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(T, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def pool_moments(moments, group=None):
    """Sum the raw accumulators [2, d_h/2, 6] over all ranks, in place; returns them.

    The counts n (field 0) add up as well, so the pooled, K-only and stream-balanced
    estimators all see the union of the ranks' calibration tokens."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(moments, op=dist.ReduceOp.SUM, group=group)
    return moments


def max_over_ranks(value: float, device=None, group=None) -> float:
    """Largest ``value`` over all ranks (used for device-timed durations)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
