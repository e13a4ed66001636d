"""The N>1 host path on CPU: two gloo ranks.

Units are independent, so splitting a batch's units over ranks (or running one
replica per rank) needs no data-path collective.  Each rank evaluates its
shard with the float64 oracle; the sum over ranks must equal the single-process
total, and the max-over-ranks timing reduction must return the largest value.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from attention_relation_kl_b200.replicas import (max_over_ranks, replica_seed, shard_units,
                                                 sum_over_ranks)


def test_shard_units_partition():
    for n in (0, 1, 5, 96, 97):
        for world in (1, 2, 3, 8):
            spans = [shard_units(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_units(4, 2, 2)
    assert replica_seed(3, 0) == 3 and replica_seed(3, 1) != replica_seed(3, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, xt, xs, out):
    import torch.distributed as dist
    from oracle import dense
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H = xt.shape[:2]
        start, stop = shard_units(B * H, world, rank)
        local = 0.0
        for u in range(start, stop):
            b, h = divmod(u, H)
            local += float(dense.fwd_unit(xt[b, h], xs[b, h])["kl"].sum())
        total = sum_over_ranks(local)
        slowest = max_over_ranks(float(rank + 1))
        out[rank] = torch.tensor([total, slowest, stop - start], dtype=torch.float64)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_units_and_reduce():
    gen = torch.Generator().manual_seed(5)
    xt = torch.randn(1, 5, 40, 8, generator=gen, dtype=torch.float64)
    xs = xt + 0.3 * torch.randn(1, 5, 40, 8, generator=gen, dtype=torch.float64)
    from oracle import dense
    ref = float(dense.fwd(xt, xs)["kl"].sum())
    out = torch.zeros(2, 3, dtype=torch.float64).share_memory_()
    mp.spawn(_worker, args=(2, _free_port(), xt, xs, out), nprocs=2, join=True)
    np.testing.assert_allclose(out[:, 0].numpy(), [ref, ref], rtol=1e-12)
    assert out[:, 1].tolist() == [2.0, 2.0]
    assert out[:, 2].tolist() == [3.0, 2.0]


def _heads_worker(rank, world, port, pairs, out):
    """One problem split by heads: each rank slices its head-range views, builds
    the descs the fused call would get, and evaluates its units with the oracle."""
    import ctypes
    import torch.distributed as dist
    from oracle import dense
    from attention_relation_kl_b200.ops import make_desc
    from attention_relation_kl_b200.replicas import shard_heads
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = shard_heads(pairs, world, rank)
        local, n_units = 0.0, 0
        for rel, (vt, vs, h0) in mine.items():
            full_t = pairs[rel][0]
            desc = make_desc(vt)
            # the view's desc: same batch stride, a head range, base moved by h0 heads
            assert (desc.B, desc.H, desc.N, desc.d) == tuple(vt.shape)
            # (a dimension of extent 1 carries stride 0 in a desc)
            for i in range(3):
                assert desc.stride[i] == (full_t.stride(i) if vt.shape[i] > 1 else 0)
            off = (vt.data_ptr() - full_t.data_ptr()) // full_t.element_size()
            assert off == h0 * full_t.stride(1)
            local += float(dense.fwd(vt, vs)["kl"].sum())
            n_units += vt.shape[0] * vt.shape[1]
        total = sum_over_ranks(local)
        units = sum_over_ranks(float(n_units))
        out[rank] = torch.tensor([total, units], dtype=torch.float64)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_split_one_problem_by_heads(world):
    import workload
    w = workload.Workload("heads", B=2, H=4, H_kv=2, N=24, d=8, dtype="fp32", causal=True,
                          relations=("q", "k", "v"), rope_base=1e4, pi_factor=4.0, v_noise=0.2,
                          seed=12)
    x = workload.generate(w)
    from oracle import dense
    ref = sum(float(dense.fwd(*x[r])["kl"].sum()) for r in w.relations)
    out = torch.zeros(world, 2, dtype=torch.float64).share_memory_()
    mp.spawn(_heads_worker, args=(world, _free_port(), x, out), nprocs=world, join=True)
    np.testing.assert_allclose(out[:, 0].numpy(), ref, rtol=1e-12)
    assert out[:, 1].tolist() == [float(w.n_units)] * world
