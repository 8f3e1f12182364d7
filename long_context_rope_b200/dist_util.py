"""Host-side helpers of the multi-GPU (weak-scaling) runs.

HGA's hot path shards by independent sequence: each rank draws and
processes its own sequence, so there is no collective on the data path.
The only cross-rank steps are a barrier around the timed region and the
max over ranks of the measured time (the slowest rank defines the step).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from .synth import seed_for_rank


def rank_seed(base_seed: int) -> int:
    r = dist.get_rank() if dist.is_available() and dist.is_initialized() else 0
    return seed_for_rank(base_seed, r)


def max_over_ranks(x: float, device="cpu") -> float:
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, seconds_max: float, world: int) -> float:
    """Aggregate throughput: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / seconds_max
