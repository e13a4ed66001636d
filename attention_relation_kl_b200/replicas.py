"""Host logic for running the relation-KL path on several GPUs of one node.

The path has no exchange step: (batch, head, relation) units are independent,
so a job either runs one replica per rank (data parallel: each rank owns its
own batch) or splits one batch's units across ranks.  Neither needs a
collective on the data path; torch.distributed is used only for a barrier,
for timing (max over ranks) and, in training, for the usual scalar loss and
weight-gradient all-reduces outside this path.
"""
from __future__ import annotations

from typing import Dict, Tuple

import torch

__all__ = ["replica_seed", "shard_units", "shard_heads", "max_over_ranks", "sum_over_ranks"]


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


def shard_heads(pairs: Dict[str, Tuple[torch.Tensor, torch.Tensor]], world: int, rank: int
                ) -> Dict[str, Tuple[torch.Tensor, torch.Tensor, int]]:
    """This rank's share of one problem: for each relation {rel: (x_t, x_s)} of
    [B, H_rel, N, d] tensors, the head range shard_units(H_rel, world, rank) as
    strided views (no copy) plus the first head's index.  Relations with no
    head on this rank are left out.  Each view is a valid desc for the fused
    calls (same B and strides, H = the range's length, base moved by h0 heads)."""
    out = {}
    for rel, (xt, xs) in pairs.items():
        h0, h1 = shard_units(int(xt.shape[1]), world, rank)
        if h1 > h0:
            out[rel] = (xt[:, h0:h1], xs[:, h0:h1], h0)
    return out


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
