"""Replica bookkeeping for one-process-per-GPU runs.

The AF-block path shards over independent units (frames of the shallow stack,
samples, whole videos of the deep flow) with no exchange between ranks: each
rank works on its own clip, the job's throughput is the units of all ranks over
the slowest rank's device time (weak scaling).  Only the timing uses a
collective (a MAX all-reduce, outside the timed region).
"""
from __future__ import annotations

import torch


def rank_seed(base: int, rank: int) -> int:
    """Seed of rank `rank`'s inputs: distinct clips per rank."""
    return base + 1000 * rank


def max_over_ranks(t: torch.Tensor, dist=None) -> torch.Tensor:
    """Element-wise max of `t` over all ranks (in place); identity without a group."""
    if dist is not None and dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t


def job_throughput(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return units_per_rank * world / seconds
