"""Host-side plumbing of the multi-GPU (weak-scaling) runs.

HGA's hot path shards by independent sequence: each rank draws and
processes its own sequence, so there is no collective on the data path.
The only cross-rank steps are a barrier around the timed region and the
max over ranks of the measured time (the slowest rank defines the step).
One process per GPU, launched by torch.distributed.run (RANK, LOCAL_RANK,
WORLD_SIZE, MASTER_ADDR / MASTER_PORT in the environment); `bench.py` runs
on this class with the NCCL backend, the CPU tests with gloo.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist

from .synth import seed_for_rank


class Dist:
    """The process group of one run. With WORLD_SIZE = 1 nothing is
    initialised and every collective is the identity."""

    def __init__(self, backend: str = "nccl", timeout_s: float = 120.0):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.device = torch.device("cpu")
        if backend == "nccl":
            self.device = torch.device("cuda", self.local if self.world > 1 else 0)
            torch.cuda.set_device(self.device)
        self.active = False
        if self.world > 1:
            kw = dict(timeout=datetime.timedelta(seconds=timeout_s))
            if backend == "nccl":
                kw["device_id"] = self.device
            dist.init_process_group(backend, **kw)
            self.active = True

    def barrier(self) -> None:
        if self.active:
            dist.barrier()

    def max(self, x: float) -> float:
        """Max of x over all ranks (every rank gets it)."""
        if not self.active:
            return float(x)
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def seed(self, base_seed: int) -> int:
        """This rank's input seed: an independent sequence per rank."""
        return seed_for_rank(base_seed, self.rank)

    def close(self) -> None:
        if self.active:
            dist.destroy_process_group()
            self.active = False


def whole_job_rate(units_per_rank: float, seconds_max: float, world: int) -> float:
    """Aggregate throughput: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / seconds_max
