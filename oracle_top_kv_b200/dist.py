"""Multi-process plumbing for running the hot path on several GPUs.

The path shards by (batch, KV group): every unit has its own K^F/V^F, index
set and query heads, and no quantity is reduced across units, so ranks never
exchange data on the data path.  What ranks do share is timing: a step's
duration is the slowest rank's, measured on each device and reduced with MAX.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def world() -> tuple:
    """(rank, world_size, local_rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, device=None, timeout_s: int = 120) -> None:
    if dist.is_initialized():
        return
    kw = dict(timeout=datetime.timedelta(seconds=timeout_s))
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def units_for_rank(n_units: int, rank: int, world_size: int) -> range:
    """Contiguous block of units [lo, hi) owned by `rank`; sizes differ by <= 1."""
    base, extra = divmod(n_units, world_size)
    lo = rank * base + min(rank, extra)
    return range(lo, lo + base + (1 if rank < extra else 0))


def max_over_ranks(value: float, device=None) -> float:
    """Largest value over all ranks (identity when not distributed)."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None) -> None:
    if dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()
