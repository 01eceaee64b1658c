"""Host-side logic of multi-GPU runs: the MLP has no exchange step on this
path, so N GPUs run N independent replicas of the workload (weak scaling).
The only cross-rank operations are a barrier and the max over ranks of the
device-timed region, done with torch.distributed (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def world():
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init(backend: str, device=None, timeout_s: int = 300) -> None:
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def barrier() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over all ranks (the slowest rank sets the time)."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, steps: int, ms_max: float, world_size: int) -> float:
    """Whole-job units per second: every rank processed `units_per_rank` per
    step, and the job took the slowest rank's time."""
    return world_size * units_per_rank * steps / (ms_max * 1e-3)
