"""Host logic for running the relation-KL path on several GPUs of one node.

The path has no exchange step: (batch, head, relation) units are independent,
so a job either runs one replica per rank (data parallel: each rank owns its
own batch) or splits one batch's units across ranks.  Neither needs a
collective on the data path; torch.distributed is used only for a barrier,
for timing (max over ranks) and, in training, for the usual scalar loss and
weight-gradient all-reduces outside this path.
"""
from __future__ import annotations

from typing import Tuple

import torch

__all__ = ["replica_seed", "shard_units", "max_over_ranks", "sum_over_ranks"]


def replica_seed(base_seed: int, rank: int) -> int:
    """Input seed of rank `rank`'s replica (rank 0 keeps the base seed)."""
    return base_seed + 1000 * rank


def shard_units(n_units: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [start, stop) range of units owned by `rank` (sizes differ by <= 1)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    q, r = divmod(n_units, world)
    start = rank * q + min(rank, r)
    return start, start + q + (1 if rank < r else 0)


def _reduce(value: float, op, device) -> float:
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks (identity without a process group)."""
    import torch.distributed as dist
    return _reduce(value, dist.ReduceOp.MAX if dist.is_available() else None, device)


def sum_over_ranks(value: float, device=None) -> float:
    """The sum of `value` over all ranks (identity without a process group)."""
    import torch.distributed as dist
    return _reduce(value, dist.ReduceOp.SUM if dist.is_available() else None, device)
