"""Request sharding across GPUs (one process per GPU).

Requests are independent at every stage of the decode path, so N GPUs split a batch
by request and exchange nothing on the data path.  This module holds the host-side
bookkeeping: which requests a rank owns, process-group setup from the launcher's
environment, and the max-over-ranks reduction used for timing.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def rank_env():
    """(rank, world_size, local_rank) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def request_range(total: int, world: int, rank: int):
    """Contiguous block of requests owned by `rank` when `total` requests are split over
    `world` ranks; sizes differ by at most one."""
    if world < 1 or not (0 <= rank < world) or total < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def init(backend: str, timeout_s: float = 120.0):
    """Join the process group described by the environment (no-op for one process)."""
    rank, world, _ = rank_env()
    if world <= 1 or dist.is_initialized():
        return dist.is_initialized()
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return True


def reduce_max(value: float, device=None) -> float:
    """Max of a scalar over all ranks (identity for one process)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
