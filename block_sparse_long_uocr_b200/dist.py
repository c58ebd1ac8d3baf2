"""One process per GPU: how decode work is split across ranks, and how times are reduced.

The decode step has no exchange between sequences: each query reads only its
own sequence's caches.  So N GPUs run N independent shards of sequences (weak
scaling: the per-GPU batch is fixed) with no collective on the data path; the
only collectives are the barrier around the timed region and the max-reduce
of the per-rank elapsed time.
"""
from __future__ import annotations

import os

import torch
import torch.distributed as dist


def env_rank_world():
    """(rank, local_rank, world_size) from the torchrun environment (1 process when unset)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def shard_range(n_total: int, rank: int, world: int):
    """Contiguous [lo, hi) share of n_total units for `rank`; shares differ by at most one."""
    base, extra = divmod(n_total, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def shard_seed(seed: int, rank: int) -> int:
    """Seed of rank's shard: different sequences on every rank, reproducible per rank."""
    return seed + 1000003 * rank


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar over the process group (identity without one)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())
