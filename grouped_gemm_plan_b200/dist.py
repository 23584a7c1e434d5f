"""Data-parallel plumbing for running the layer on several GPUs of one node.

Tokens are independent and every GPU holds all experts, so N GPUs run N
independent batches: rank r processes its own batch (same shape, its own seed)
and nothing is exchanged on the data path.  The only collectives are the barrier
around a timed region and the max over ranks of the measured device times
(torch.distributed: NCCL on GPUs, gloo in the CPU tests).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist

from .workload import Workload, rank_workload


def env_rank() -> tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment (1 process: 0, 0, 1)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init(backend: str, timeout_s: float = 120.0, device: torch.device | None = None) -> bool:
    """Join the process group when WORLD_SIZE > 1; returns whether a group exists."""
    rank, _, world = env_rank()
    if world <= 1:
        return False
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)
    return True


def shard(wl: Workload, rank: int) -> Workload:
    """The batch a rank runs: the same shape with its own seed (rank 0 keeps the base seed)."""
    return rank_workload(wl, rank)


def barrier(device: torch.device | None = None) -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
    if device is not None and device.type == "cuda":
        torch.cuda.synchronize(device)


def max_over_ranks(values: list[float], device: torch.device | None = None) -> list[float]:
    """Element-wise max of per-rank measurements (identity on one process)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def whole_job_rate(units_per_rank: int, world: int, seconds_max: float) -> float:
    """Units all ranks processed divided by the slowest rank's time."""
    return world * units_per_rank / seconds_max


def finish() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
