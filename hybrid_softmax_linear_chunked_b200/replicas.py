"""One process per GPU, each running its own replica of the workload.

The hybrid attention forward has no exchange step: every (batch, head) pair is an independent
problem (the chunk recurrence runs along the sequence of one head), so N GPUs process N
batches with no collective on the data path.  The process group only carries the timing
barrier and the max-over-ranks reduction of the measured times.

Ranks read RANK / WORLD_SIZE / LOCAL_RANK from the environment set by torchrun and rendezvous
at MASTER_ADDR (127.0.0.1 by default).  Every rank takes the same collective steps in the same
order; the group has a short timeout so that ranks waiting for a dead peer end with an error.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass


@dataclass
class Replicas:
    rank: int = 0
    world: int = 1
    local_rank: int = 0
    backend: str | None = None
    _dist: object = None

    @staticmethod
    def from_env(backend: str, timeout_s: float = 120.0) -> "Replicas":
        """Join the process group when WORLD_SIZE > 1; a single process needs none."""
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        local = int(os.environ.get("LOCAL_RANK", "0"))
        if world <= 1:
            return Replicas(rank, world, local)
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        if backend == "nccl":
            import torch
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
        return Replicas(rank, world, local, backend, dist)

    @property
    def distributed(self) -> bool:
        return self._dist is not None

    def seed(self, base: int) -> int:
        """Each replica draws its own batch: seed base + rank."""
        return base + self.rank

    def barrier(self) -> None:
        if self._dist is not None:
            self._dist.barrier()

    def max(self, x: float, device=None) -> float:
        """Max of a float over ranks (the job time is the slowest rank's)."""
        if self._dist is None:
            return float(x)
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=device)
        self._dist.all_reduce(t, op=self._dist.ReduceOp.MAX)
        return float(t.item())

    def all_values(self, x: float, device=None) -> list[float]:
        """The float of every rank, in rank order."""
        if self._dist is None:
            return [float(x)]
        import torch
        t = torch.zeros(self.world, dtype=torch.float64, device=device)
        t[self.rank] = float(x)
        self._dist.all_reduce(t, op=self._dist.ReduceOp.SUM)
        return [float(v) for v in t.tolist()]

    def close(self) -> None:
        if self._dist is not None:
            self._dist.barrier()
            self._dist.destroy_process_group()
            self._dist = None


def job_throughput(units_per_rank: float, world: int, max_ms_per_step: float) -> float:
    """Whole-job throughput: the units all ranks processed per second of the slowest rank."""
    return units_per_rank * world / (max_ms_per_step * 1e-3)
