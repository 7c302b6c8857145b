"""Multi-GPU plumbing for the row-parallel MXNorm path (host side only).

MXNorm is row-local (gist.science, "MXNorm: Reusing MXFP block scales for
efficient tensor normalisation", technical summary section 2.1: every statistic
is taken along one row's hidden dimension), so rows shard across ranks with no
exchange in the forward.  The backward's gamma gradient is a sum over rows
(section 2.3), i.e. an ordinary data-parallel gradient all-reduce.

These helpers hold no arithmetic of the method; they partition rows and run
torch.distributed collectives (NCCL on GPUs, gloo on the CPU in tests).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def row_range(T: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous rows [lo, hi) of rank `rank`: sizes differ by at most one."""
    if world <= 0 or not (0 <= rank < world) or T < 0:
        raise ValueError("bad partition arguments")
    base, extra = divmod(T, world)
    lo = rank * base + min(rank, extra)
    hi = lo + base + (1 if rank < extra else 0)
    return lo, hi


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks (1 rank: the value itself)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t[0])


def allreduce_dgamma(dgamma_partial: torch.Tensor) -> torch.Tensor:
    """Sum of every rank's gamma-gradient partial (in place; fp32 or fp64)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(dgamma_partial, op=dist.ReduceOp.SUM)
    return dgamma_partial
