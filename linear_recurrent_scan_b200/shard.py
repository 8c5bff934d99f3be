"""Data-parallel plumbing for the recurrence: (batch, head) units are independent,
so ranks split the batch with no data-path collective.  torch.distributed is only
used for barriers and for reducing timings (max over ranks)."""
from __future__ import annotations

from typing import Tuple

import torch


def batch_range(global_batch: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [start, stop) slice of the batch owned by `rank`; the first
    `global_batch % world` ranks take one extra sequence."""
    if world < 1 or not 0 <= rank < world or global_batch < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank scalar (e.g. elapsed device time) over all ranks."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def all_reduce_sum_(tensors) -> None:
    """In-place sum over ranks of parameter gradients (the backward pass's dA and
    dD, which sum over the batch): the one exchange that data-parallel training adds.
    A no-op on a single rank.  Every rank must pass the same tensors in the same order."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return
    for t in tensors:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
