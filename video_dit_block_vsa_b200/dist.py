"""Process-group plumbing for running the VSA path on several GPUs of one node.

The path needs no exchange between GPUs: every (batch, head) is independent, so
each rank runs its own batch (weak scaling) and the ranks only meet for a
barrier around the timed region and for the max-over-ranks of the measured time.
One process per GPU; rank, world size and master address come from the
environment variables torchrun sets.
"""

from __future__ import annotations

import os
from dataclasses import dataclass
from datetime import timedelta

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local_rank: int


def rank_info() -> RankInfo:
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 300.0) -> RankInfo:
    """Initialises the default process group when the world has several ranks."""
    info = rank_info()
    if info.world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s))
    return info


def barrier(info: RankInfo) -> None:
    if info.world > 1:
        dist.barrier()


def max_over_ranks(value: float, info: RankInfo, device=None) -> float:
    """The largest value any rank holds (the job's time is its slowest rank's)."""
    if info.world == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, steps: int, max_elapsed_ms: float, world: int) -> float:
    """Whole-job throughput: units every rank processed / the slowest rank's time (per s)."""
    return world * units_per_rank * steps / (max_elapsed_ms * 1e-3)


def shutdown(info: RankInfo) -> None:
    if info.world > 1 and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
