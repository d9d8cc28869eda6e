"""Data-parallel replicas: sequences are independent, so N GPUs run N engines.

There is no collective on the data path.  The only cross-rank steps are the
sequence assignment and the max-over-ranks reduction of the timed region.
"""

from __future__ import annotations

from typing import List, Optional


def shard_ids(rank: int, world: int, per_rank: int) -> List[int]:
    """Sequence ids of one rank: rank r owns ids r*per_rank .. r*per_rank + per_rank - 1."""
    if not (0 <= rank < world) or per_rank < 1:
        raise ValueError((rank, world, per_rank))
    return [rank * per_rank + i for i in range(per_rank)]


def max_over_ranks(value: float, device: Optional[str] = None) -> float:
    """The largest `value` over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_lists(items: list) -> list:
    """All ranks' lists concatenated in rank order (identity without a process group)."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return list(items)
    out = [None] * dist.get_world_size()
    dist.all_gather_object(out, items)
    return [x for part in out for x in part]
