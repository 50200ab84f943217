"""Multi-process plumbing: one process per GPU, one shard of a problem per rank.

Every (batch, head) slice of LSH attention is independent through hashing,
sorting, chunk attention, the round combine and the backward pass, so a
problem is split across ranks by contiguous ranges of its B*H slices
(``shard``) and each rank runs its range through the C ABI as a problem of
its own (the slices are contiguous in the [B, H, L, d] layout). Ranks share
no data; the only collective is the max-over-ranks reduction of the
measured time.
"""
from __future__ import annotations

import datetime
import os
from typing import Tuple

import torch
import torch.distributed as dist


def env_rank() -> Tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str, timeout_s: float = 120.0) -> Tuple[int, int, int]:
    rank, local, world = env_rank()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=timeout_s))
    return rank, local, world


def shard(n: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [lo, hi) share of n independent slices for ``rank``."""
    q, r = divmod(n, world)
    lo = rank * q + min(rank, r)
    return lo, lo + q + (1 if rank < r else 0)


def max_over_ranks(x: float, device=None) -> float:
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def finish():
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
