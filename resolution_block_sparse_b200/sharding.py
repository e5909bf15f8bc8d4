"""Host-side logic of the multi-GPU path: (batch, head) shards, no collective.

Every (batch, head) slice of the MRA-2 forward pass is independent (pooling,
selection, attention and combine never cross heads), so N ranks split a job
of independent slices with no data-path communication.  The only collective
is for measurement: the max over ranks of a device-timed duration.
"""
from __future__ import annotations

from typing import Tuple


def shard_range(units: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [start, stop) of `units` owned by `rank`; sizes differ by at
    most one and every unit is owned by exactly one rank."""
    if world < 1 or not (0 <= rank < world) or units < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(units, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def weak_scaling_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s shard when every rank holds a full-size batch of
    its own (weak scaling): distinct, reproducible per rank."""
    return base_seed + 7919 * rank


def max_over_ranks(values, device=None):
    """Element-wise max over ranks of a list of floats (torch.distributed
    all-reduce, any backend); returns the list unchanged with one rank."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]
