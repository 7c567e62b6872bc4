"""Data-parallel plumbing over torch.distributed (one process per GPU).

Every (b, h) pair of the recurrence is independent, so ranks shard the batch
with no exchange inside the forward or backward kernels.  The one exchange is
the gradient of the shared per-head W: dW is a sum over the global batch, so
each rank's dW (already summed over its own batch rows) is all-reduced.
"""
from __future__ import annotations

import datetime
import os

import torch


def init(backend: str, timeout_s: int = 120):
    """Initialises the default process group from the torchrun environment
    (RANK, WORLD_SIZE, MASTER_ADDR, MASTER_PORT); returns (rank, world)."""
    import torch.distributed as dist
    if not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist.get_rank(), dist.get_world_size()


def world_from_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))


def allreduce_dW(dW: torch.Tensor) -> torch.Tensor:
    """In-place sum of the per-rank dW over all ranks (no-op on one rank)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(dW, op=dist.ReduceOp.SUM)
    return dW


def max_over_ranks(x: float, device=None) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
