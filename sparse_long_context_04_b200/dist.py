"""Multi-process plumbing for running the DSA decode step on several GPUs.

Decode sequences are independent, so each process (one per GPU) runs its own
batch: there is no collective on the data path. The only collectives are the
benchmark's barrier and the max over ranks of the timed region.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def rank_info():
    """(world_size, rank, local_rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, device=None, timeout_s: int = 300) -> None:
    """Join the process group when launched with more than one rank."""
    world, _, _ = rank_info()
    if world > 1 and not dist.is_initialized():
        kw = {"device_id": device} if device is not None and backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def barrier() -> None:
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """The largest value over all ranks (the job's time is its slowest rank's)."""
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank decodes a different synthetic batch of the same shape."""
    return base_seed + 1000 * rank


def job_rate(world: int, rows_per_rank: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: rows decoded by all ranks per second of the slowest rank."""
    return world * rows_per_rank * steps / (max_ms / 1e3)


def finish() -> None:
    if dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
