"""Multi-GPU plumbing of the hot path (one process per GPU, torch.distributed).

The block is row-independent: RMSNorm, SwiGLU and the cross-entropy are per
token, so N GPUs run N independent batches (data parallel, weak scaling) with
no collective on the data path.  The only collectives are for measurement: a
barrier around the timed region and the max over ranks of the device time.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env():
    """(world_size, rank, local_rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 300):
    """Initialise the process group when launched with more than one rank."""
    ws, rank, local = env()
    if ws > 1 and not dist.is_initialized():
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return ws, rank, local


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's own batch (each rank draws different tokens)."""
    return base + 1000 * rank


def barrier():
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """The largest of every rank's value (device time of the timed region)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(work_per_rank_per_step: float, steps: int, max_seconds: float, world: int) -> float:
    """Whole-job throughput: the work of all ranks divided by the slowest rank's time."""
    return world * work_per_rank_per_step * steps / max_seconds


def shutdown():
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
