"""Host plumbing of a multi-GPU run: one process per GPU, launched by
torchrun.  The indexer shards without an exchange step (prefill rows are
independent given the keys, decode requests are independent), so each rank
works on its own batch and the only collectives are the barrier around the
timed region and the max over ranks of the measured time."""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env():
    """(rank, world_size, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 300):
    rank, world, local = env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world, local


def barrier(device=None):
    if dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    """The max of a per-rank scalar (a device time) over all ranks."""
    if not (dist.is_initialized() and dist.get_world_size() > 1):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int, base: int = 0) -> int:
    """Seed of the rank's own synthetic batch (weak scaling: fixed work per rank)."""
    return base + rank


def finish():
    if dist.is_initialized():
        dist.destroy_process_group()
