"""Multi-GPU by sequence sharding: one process per GPU, no data-path exchange.

Decode and prefill are independent per sequence (and per head), so a batch is
split across ranks by sequence and every rank runs the unchanged kernels on its
own shard; the only collective is the timing reduction (max over ranks). The
functions work with any torch.distributed backend (NCCL on GPUs, gloo in the
CPU tests).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_rank() -> tuple[int, int, int]:
    """(world_size, rank, local_rank) from the torchrun environment (1, 0, 0 without it)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0, device: torch.device | None = None) -> None:
    """Initialise the default process group from the environment, with a short timeout."""
    if dist.is_initialized():
        return
    kw = {"device_id": device} if device is not None and backend == "nccl" else {}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def shard(total: int, world: int, rank: int) -> range:
    """The contiguous range of sequences rank `rank` owns when `total` are split over `world` ranks
    (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of {world}")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def barrier() -> None:
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(value: float, device: torch.device | str = "cpu") -> float:
    """The largest `value` over all ranks (the job's time is its slowest rank's)."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device: torch.device | str = "cpu") -> float:
    """Sum of `value` over all ranks (units processed by the whole job)."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shutdown() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()
