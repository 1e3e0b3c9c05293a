"""Data-parallel placement of request rows over GPUs.

The draft round is independent per request row (every step is per row:
context K/V, attention over the row's own cache, the walk), so N GPUs each
hold the full weights and serve a contiguous share of the rows; no
collective runs on the data path. Only timing and results are gathered.
"""
from __future__ import annotations

from typing import Tuple


def shard_rows(A: int, world: int, rank: int) -> Tuple[int, int]:
    """Rows [lo, hi) of A request rows served by `rank` of `world` (sizes differ by at most one)."""
    if world <= 0 or not 0 <= rank < world or A < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(A, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, group=None) -> float:
    """The largest of one float per rank (the job's time is its slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return float(value)
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
