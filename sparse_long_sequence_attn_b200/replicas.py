"""Host plumbing for running the forward on several GPUs of one node.

The forward has no exchange step between problems: every (batch, head,
position range) is independent, so N GPUs run N independent replicas of a
workload (each its own seeded inputs) with no collective on the data path.
The only collectives are the timing barrier and the max-over-ranks of the
timed region, done with torch.distributed (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

import os

import torch
import torch.distributed as dist


def dist_env():
    """(world_size, rank, local_rank) from the torch.distributed launcher's env."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_seed(base_seed: int, rank: int) -> int:
    """Seed of rank's replica: distinct per rank, rank 0 keeps the base seed."""
    return base_seed + 7919 * rank


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over the default process group (identity when
    no group is initialised)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank: float, world_size: int, max_seconds: float) -> float:
    """Whole-job throughput: units all ranks processed over the slowest rank's time."""
    return units_per_rank * world_size / max_seconds
