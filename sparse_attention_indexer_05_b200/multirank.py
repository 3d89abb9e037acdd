"""Host plumbing of a multi-GPU run: one process per GPU, launched by
torchrun.  The indexer shards without an exchange step (prefill rows are
independent given the keys, decode requests are independent), so the only
collectives are the barrier around the timed region and the max over ranks
of the measured time.  Two ways to use N GPUs:
  * independent batches: each rank works on its own batch (weak scaling);
  * one request split across ranks (strong scaling): every rank holds the
    request's keys, queries and weights (the keys are what every row needs;
    here each rank generates or copies them whole, no collective), and
    computes the top-k of the rows zigzag_ranges() gives it, through the
    library's row-range entry points; the ranks' rows are disjoint and
    together cover the request."""
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


def zigzag_ranges(n: int, world: int, rank: int, align: int = 1):
    """Rows of one request of n tokens that `rank` owns when the request is
    split over `world` ranks: the request is cut into 2*world chunks of equal
    length, at multiples of `align` (a multiple of the PIVOT group size keeps
    every group on one rank), and rank r owns chunks r and 2*world-1-r.  Under
    the causal mask a chunk's work grows with its position, so each rank's
    early chunk and late chunk add up to the same work on every rank, up to
    the alignment.  Returns the rank's non-empty request-local ranges
    [(lo, hi), ...] in ascending order."""
    if world < 1 or not 0 <= rank < world or align < 1 or n < 0:
        raise ValueError("bad split arguments")
    nch = 2 * world
    bounds = [min(n, int(round(c * n / nch / align)) * align) for c in range(nch)] + [n]
    out = []
    for c in sorted((rank, nch - 1 - rank)):
        lo, hi = bounds[c], bounds[c + 1]
        if hi > lo:
            out.append((lo, hi))
    return out


def causal_pairs(ranges) -> int:
    """(query, key) pairs under the causal mask of the rows in `ranges`."""
    return sum((hi * (hi + 1) - lo * (lo + 1)) // 2 for lo, hi in ranges)
