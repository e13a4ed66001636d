"""Row-sharded (context-parallel) relation KL over the ranks of a process group.

For sequences too long for one GPU's time budget, every rank holds a
contiguous shard of the tokens and the ranks split the rows of every
(batch, head, relation) unit between them.  The pages state the method for
one device (LinearARD: pith.science verdict page, pith_extraction.
key_machinery, Phase 1 / Phase 2); the split rests on two facts of that
computation: a row's statistics and KL need only that row's logits (every
column), and dX_s = s (G + G^T) X_s is a sum of independent per-row terms.

One step, per group of relations (Q, K, V of a layer):

1. all-gather the teacher and student token shards: every rank sees every
   column tile (X is O(N) memory);
2. forward of this rank's part of every unit's work items
   (relkl_fwd_qkv_part), into zeroed kl / stats buffers;
3. all-reduce (sum) kl and stats: every rank then holds every row's
   statistics, which the backward's items need;
4. backward of the same part (relkl_bwd_qkv_part): the contributions of
   this rank's rows of G to both sides of dX_s;
5. reduce-scatter (sum) dX_s over the token shards: each rank receives the
   gradient of its own tokens.

Layout: token shards are token-major, [n_local, B, H, d] (the gathered tensor
[N, B, H, d] is handed to the kernels as a strided [B, H, N, d] view, so no
copy is made).  The parts are the library's own (items part, part + W, ...
of every unit), so each rank holds nearly equal causal work.

The collectives are torch.distributed calls (NCCL on GPUs, gloo on CPU for
the tests); the two compute steps are injectable so that the host logic can
be exercised on CPU ranks.  No peer memory is handed to any kernel and no
load uses multicast.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

__all__ = ["gather_tokens", "cp_forward", "cp_backward", "context_parallel_step",
           "library_fwd_part", "library_bwd_part"]

Pair = Tuple[torch.Tensor, torch.Tensor]


def _world(group) -> Tuple[int, int]:
    if not dist.is_available() or not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def gather_tokens(local: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather token-major shards [n, ...] into [world * n, ...] (rank order)."""
    world, _ = _world(group)
    if world == 1:
        return local
    local = local.contiguous()
    out = torch.empty((world * local.shape[0],) + tuple(local.shape[1:]), dtype=local.dtype,
                      device=local.device)
    if local.is_cuda:
        dist.all_gather_into_tensor(out, local, group=group)
    else:
        dist.all_gather(list(out.chunk(world, dim=0)), local, group=group)
    return out


def _reduce_scatter_tokens(full_bhnd: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """Sum [B, H, N, d] over ranks and return this rank's token shard, token-major
    [N / world, B, H, d]."""
    B, H, N, d = full_bhnd.shape
    n = N // world
    # token-major chunks, one per rank: [world, n, B, H, d]
    chunks = full_bhnd.view(B, H, world, n, d).permute(2, 3, 0, 1, 4).contiguous()
    if world == 1:
        return chunks[0]
    out = torch.empty((n, B, H, d), dtype=full_bhnd.dtype, device=full_bhnd.device)
    if full_bhnd.is_cuda:
        dist.reduce_scatter_tensor(out, chunks.view(world * n, B, H, d), group=group)
    else:
        # gloo has no reduce-scatter: reduce every chunk to its owner
        _, rank = _world(group)
        for r in range(world):
            buf = chunks[r].clone()
            dist.reduce(buf, dst=dist.get_global_rank(group, r) if group is not None else r,
                        group=group)
            if r == rank:
                out.copy_(buf)
    return out


def library_fwd_part(pairs: Sequence[Pair], causal: bool, scale: float, part: Tuple[int, int]):
    """Forward of one part through librelkl.so: [(kl, stats)] per relation, zero
    on the rows of other parts."""
    from . import ops
    return ops.relkl_fwd_qkv(pairs, causal, scale, part=part)


def library_bwd_part(pairs: Sequence[Pair], stats: Sequence[torch.Tensor], causal: bool,
                     scale: float, part: Tuple[int, int]) -> List[torch.Tensor]:
    """Backward of one part through librelkl.so: this part's share of dX_s."""
    from . import ops
    return ops.relkl_bwd_qkv(pairs, stats, None, causal, scale, part=part)


def cp_forward(local_pairs: Sequence[Pair], causal: bool = True, scale: float = 0.0, group=None,
               fwd_part: Optional[Callable] = None):
    """Steps 1-3: gather the token shards, run this rank's part of the forward
    and combine every part's kl and statistics.  Returns (full_pairs, kl,
    stats): the gathered [B, H, N, d] views (for cp_backward) and kl [B, H, N],
    stats [B, H, N, 4] of every row, per relation."""
    world, rank = _world(group)
    fwd_part = fwd_part or library_fwd_part
    full = []
    for xt, xs in local_pairs:
        if xt.shape != xs.shape or xt.dim() != 4:
            raise ValueError("token shards must be matching [n_local, B, H, d] tensors")
        gt = gather_tokens(xt, group).permute(1, 2, 0, 3)      # [B, H, N, d] view
        gs = gather_tokens(xs, group).permute(1, 2, 0, 3)
        full.append((gt, gs))
    outs = fwd_part(full, causal, scale, (rank, world))
    kl = [o[0] for o in outs]
    stats = [o[1] for o in outs]
    if world > 1:
        for t in kl + stats:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return full, kl, stats


def cp_backward(full_pairs: Sequence[Pair], stats: Sequence[torch.Tensor], causal: bool = True,
                scale: float = 0.0, group=None, bwd_part: Optional[Callable] = None):
    """Steps 4-5: this rank's part of the backward, then the reduce-scatter of
    dX_s over the token shards.  Returns this rank's [n_local, B, H, d] float32
    shard of dX_s per relation."""
    world, rank = _world(group)
    bwd_part = bwd_part or library_bwd_part
    dxs = bwd_part(full_pairs, stats, causal, scale, (rank, world))
    return [_reduce_scatter_tokens(dx, world, group) for dx in dxs]


def context_parallel_step(local_pairs: Sequence[Pair], causal: bool = True, scale: float = 0.0,
                          group=None, fwd_part: Optional[Callable] = None,
                          bwd_part: Optional[Callable] = None):
    """One forward + backward of 1..3 relations with rows split over the group.

    ``local_pairs``: per relation, this rank's (teacher, student) token shards,
    token-major [n_local, B, H, d], equal n_local on every rank.
    Returns (kl, stats, dx_local): kl [B, H, N] and stats [B, H, N, 4] of
    every row (identical on every rank) and this rank's token shard of dX_s,
    [n_local, B, H, d] float32, per relation.  The backward's upstream
    gradient is the default 1/N per row (the gradient of the per-unit mean).
    """
    full, kl, stats = cp_forward(local_pairs, causal, scale, group, fwd_part)
    dx_local = cp_backward(full, stats, causal, scale, group, bwd_part)
    return kl, stats, dx_local
