"""Multi-GPU plumbing for the benchmark: one process per GPU, independent
replicas of the workload (the LC-VQ hot path has no exchange step, so there is
no collective in the data path).  Only the timing is combined: every rank's
device time is reduced with MAX, and throughput counts the units all ranks
processed.

Works with NCCL on GPUs and with gloo on CPU (the tests run two gloo ranks).
"""

from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


class Replicas:
    def __init__(self, backend: str | None = None, timeout_s: int = 120):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        if self.backend == "nccl":
            torch.cuda.set_device(self.local if self.world > 1 else 0)
            self.dev = torch.device("cuda", torch.cuda.current_device())
        else:
            self.dev = torch.device("cpu")
        self.owns_group = False
        if self.world > 1 and not dist.is_initialized():
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=timeout_s))
            self.owns_group = True

    def barrier(self):
        if self.world > 1:
            dist.barrier()

    def max(self, x: float) -> float:
        """Max over ranks of a per-rank float (the slowest rank's time)."""
        if self.world == 1:
            return float(x)
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def sum(self, x: float) -> float:
        if self.world == 1:
            return float(x)
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.dev)
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.owns_group and dist.is_initialized():
            dist.destroy_process_group()


def throughput(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: units processed by all ranks / slowest rank's time."""
    return units_per_rank * world / max_seconds


def shard(n_items: int, world: int, rank: int) -> range:
    """Contiguous, balanced share of n_items for one rank (used when a
    workload is partitioned instead of replicated)."""
    lo = n_items * rank // world
    hi = n_items * (rank + 1) // world
    return range(lo, hi)
