"""Host plumbing for running the path as N independent replicas, one process per GPU.

The attention path has no exchange step on one GPU and none between GPUs: every rank
runs the same workload on its own device. The only collectives are the timing barrier
and the max over ranks of the device-measured time, so the whole-job throughput is
N x (work per rank) / (slowest rank's time) -- weak scaling.
"""
from __future__ import annotations

import datetime
import os


class Replicas:
    """Rank bookkeeping read from the launcher's environment (RANK / LOCAL_RANK /
    WORLD_SIZE / MASTER_ADDR / MASTER_PORT), with a process group when WORLD_SIZE > 1."""

    def __init__(self, backend: str = "nccl", timeout_s: float = 120.0):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self._dist = None
        if self.world > 1:
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
            self._dist = dist

    def barrier(self) -> None:
        if self._dist is not None:
            self._dist.barrier()

    def max_over_ranks(self, x: float, device=None) -> float:
        """Largest x over all ranks (every rank gets it)."""
        if self._dist is None:
            return float(x)
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=device)
        self._dist.all_reduce(t, op=self._dist.ReduceOp.MAX)
        return float(t.item())

    def aggregate_throughput(self, work_per_rank: float, seconds_per_rank: float, device=None) -> float:
        """Whole-job throughput: world x work_per_rank / (max over ranks of seconds)."""
        slowest = self.max_over_ranks(seconds_per_rank, device)
        return self.world * work_per_rank / slowest if slowest > 0 else 0.0

    def close(self) -> None:
        if self._dist is not None:
            self._dist.destroy_process_group()
            self._dist = None
