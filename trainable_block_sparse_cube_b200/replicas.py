"""Host-side coordination of independent replicas (one process per GPU).

Every (batch, head) slice of the forward pass is independent, so the
multi-GPU form has no exchange step: N processes run the same workload on
their own GPUs. Only the measurement is shared: a barrier on both sides of
the timed region, the elapsed time taken as the maximum over ranks, and the
whole-job throughput = N x per-rank work / that maximum. Rank 0 reports.

The process group uses NCCL on GPUs and gloo on CPU (tests); its timeout is
short so that a rank that fails ends the others' next collective with an
error instead of a hang.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

import torch


@dataclass
class Replicas:
    rank: int
    world: int
    local_rank: int
    backend: str | None  # None for a single process

    @property
    def is_reporter(self) -> bool:
        return self.rank == 0

    def _device(self):
        return torch.device("cuda", torch.cuda.current_device()) if self.backend == "nccl" else torch.device("cpu")

    def barrier(self) -> None:
        if self.backend is not None:
            torch.distributed.barrier()

    def max_over_ranks(self, x: float) -> float:
        """The largest of the ranks' values of x (x itself for one process)."""
        if self.backend is None:
            return float(x)
        t = torch.tensor([float(x)], dtype=torch.float64, device=self._device())
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())

    def job_throughput(self, work_per_rank: float, t_max_s: float) -> float:
        """Whole-job rate: every rank did work_per_rank in at most t_max_s."""
        return self.world * work_per_rank / t_max_s

    def close(self) -> None:
        if self.backend is not None and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


def from_env(backend: str = "nccl", timeout_s: float = 120.0) -> Replicas:
    """Reads RANK / WORLD_SIZE / LOCAL_RANK (set by torch.distributed.run) and,
    for more than one process, joins the process group."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world <= 1:
        return Replicas(rank, 1, local, None)
    torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return Replicas(rank, world, local, backend)
