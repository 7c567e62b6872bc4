"""Multi-GPU plumbing over torch.distributed (one process per GPU).

Every (b, h) pair of the recurrence is independent, so ranks can shard it
two ways with no exchange inside the forward or backward kernels:
* the batch (data parallel): the one exchange is the gradient of the shared
  per-head W, a sum over the global batch, so each rank's dW (already summed
  over its own batch rows) is all-reduced (allreduce_dW);
* the heads, a whole number of k / q head groups per rank (the topology-aware
  tensor-parallel strategy of the pages, gist.science technical summary §2.2):
  a rank holds its groups' k and q and their heads' v, f, W and state, so
  nothing at all is exchanged (head_shard).
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


def head_shard(x: dict, rank: int, world: int) -> dict:
    """The part of a problem that rank `rank` of `world` holds when heads are
    sharded: head groups [r·G/N, (r+1)·G/N) of k, q (and dk, dq) and the heads
    of those groups of every per-head tensor (v, f, W, H0, HT, dY, y, dv, df,
    dW, dH0, ckpt).  G is k's head count (= H when k and q are per head) and
    must be a multiple of world.  Returns contiguous slices; None stays None."""
    G, H = x["k"].shape[1], x["v"].shape[1]
    if G % world or H % G:
        raise ValueError("%d k/q head groups of %d heads cannot be split over %d ranks" % (G, H, world))
    g0, g1 = rank * G // world, (rank + 1) * G // world
    h0, h1 = g0 * (H // G), g1 * (H // G)
    group_dim1 = ("k", "q", "dk", "dq")
    head_dim0 = ("W", "dW")
    out = {}
    for n, t in x.items():
        if t is None:
            out[n] = None
        elif n in group_dim1:
            out[n] = t[:, g0:g1].contiguous()
        elif n in head_dim0:
            out[n] = t[h0:h1].contiguous()
        else:
            out[n] = t[:, h0:h1].contiguous()
    return out
