"""Data-parallel replicas of the MoE layer, one process per GPU.

The layer has no exchange step between GPUs: with replicated experts each rank
routes, dispatches and computes its own batch of tokens. The only collectives
are around measurement: a barrier on each side of a timed region, and the
maximum of the ranks' durations, so whole-job throughput is the tokens all
ranks processed divided by the slowest rank's time.

Ranks come from the launcher's environment (RANK, WORLD_SIZE, LOCAL_RANK), as
``torch.distributed.run`` sets them. The process group gets a short timeout,
so a rank that fails or never arrives ends the others' next collective with an
error instead of a hang.
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
    local: int

    @property
    def distributed(self) -> bool:
        return self.world > 1


def rank_info() -> RankInfo:
    """This process's rank, world size and local rank (1-process defaults)."""
    return RankInfo(int(os.environ.get("RANK", "0")),
                    int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: float = 120.0,
         device: torch.device | None = None) -> RankInfo:
    """Join the process group when there is more than one rank."""
    info = rank_info()
    if info.distributed and not dist.is_initialized():
        kw = {"device_id": device} if device is not None and device.type == "cuda" else {}
        dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s), **kw)
    return info


def batch_seed(seed: int, info: RankInfo) -> int:
    """Seed of this rank's batch: every replica works on different tokens."""
    return int(seed) + info.rank


def barrier(info: RankInfo) -> None:
    if info.distributed:
        dist.barrier()


def max_over_ranks(value: float, info: RankInfo,
                   device: torch.device | None = None) -> float:
    """The largest of the ranks' values (a duration), on every rank."""
    if not info.distributed:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else torch.device("cpu"))
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_step: int, steps: int, info: RankInfo,
                   slowest_ms: float) -> float:
    """Tokens per second of the whole job: all ranks' tokens over the slowest
    rank's time (weak scaling: each rank's batch is fixed)."""
    if slowest_ms <= 0:
        raise ValueError("duration must be positive")
    return info.world * steps * tokens_per_step / (slowest_ms / 1e3)


def finalize(info: RankInfo) -> None:
    if info.distributed and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
