"""Data-parallel replicas for the benchmark: one process per GPU, each running
its own copy of the workload (windows are independent, so ranks exchange
nothing on the data path). Only the timing is combined: the job's time is
the slowest rank's, the job's work is the sum over ranks.
"""

from __future__ import annotations

import os
from datetime import timedelta

import torch
import torch.distributed as dist


def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0):
    """Initialise the process group from torchrun's environment (no-op for one process)."""
    rank, world, _ = env_rank()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=timeout_s))
    return rank, world


def barrier(device=None):
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def combine(elapsed_s: float, units: float, device=None):
    """(max elapsed over ranks, sum of units over ranks, world size)."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(elapsed_s), float(units), 1
    dev = device if (device is not None and dist.get_backend() == "nccl") else torch.device("cpu")
    t = torch.tensor([elapsed_s], dtype=torch.float64, device=dev)
    u = torch.tensor([units], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item()), dist.get_world_size()


def shutdown():
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
