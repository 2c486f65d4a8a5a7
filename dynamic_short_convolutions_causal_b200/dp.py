"""Data-parallel plumbing for the low-rank dynamic short convolution.

Sequences are independent, so a batch shards across ranks by sequence with no
exchange in the forward or in dx / dz.  The one cross-rank step of a data-parallel
training step is the weight gradient of the low-rank factor: dU sums over every
token of the global batch (dU[r,j] = sum_{b,t} z[b,t,r] dw[b,t,j]), so each rank's
dU is summed across ranks.  These helpers use torch.distributed (NCCL on GPUs, gloo
on CPU); they do no arithmetic of the method themselves.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_sequences(B: int, rank: int, world: int) -> range:
    """Sequences of a global batch of B owned by `rank` (contiguous, as even as possible)."""
    lo = B * rank // world
    hi = B * (rank + 1) // world
    return range(lo, hi)


def allreduce_weight_grad(dU: torch.Tensor) -> torch.Tensor:
    """Sum the per-rank dU in place across the process group (no-op on one rank)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(dU, op=dist.ReduceOp.SUM)
    return dU


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks (step times are reported as the slowest rank's)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
