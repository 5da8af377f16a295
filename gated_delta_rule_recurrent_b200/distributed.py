"""Multi-GPU plumbing for the decode step: one process per GPU, no data-path
collective.

Every (item, value head) of the decode step is independent, so N GPUs simply
decode N independent batches, each with its own state pool (weak scaling).
The only cross-rank traffic is timing bookkeeping: a barrier around the timed
region, the maximum of the per-rank elapsed times, and the sum of the units
processed. These helpers work with any torch.distributed backend (NCCL on
GPUs, gloo on CPU for tests).
"""
from __future__ import annotations

import os
from typing import Optional, Tuple

import torch
import torch.distributed as dist

__all__ = ["rank_env", "rank_seed", "max_over_ranks", "sum_over_ranks", "throughput"]


def rank_env() -> Tuple[int, int, int]:
    """(world size, rank, local rank) from the launcher's environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank ``rank``'s batch: distinct per rank, equal to ``base_seed`` on rank 0."""
    return base_seed + 7919 * rank


def _reduce(value: float, op, device: Optional[torch.device]) -> float:
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(value: float, device: Optional[torch.device] = None) -> float:
    """The maximum of ``value`` over all ranks (the value itself without a process group)."""
    return _reduce(value, dist.ReduceOp.MAX, device)


def sum_over_ranks(value: float, device: Optional[torch.device] = None) -> float:
    """The sum of ``value`` over all ranks (the value itself without a process group)."""
    return _reduce(value, dist.ReduceOp.SUM, device)


def throughput(local_units: float, local_seconds: float,
               device: Optional[torch.device] = None) -> Tuple[float, float]:
    """Whole-job throughput: units processed by all ranks over the slowest rank's time.

    Returns (units per second, slowest time in seconds).
    """
    units = sum_over_ranks(local_units, device)
    seconds = max_over_ranks(local_seconds, device)
    return units / seconds, seconds
