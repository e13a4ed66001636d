"""Row-sharded (context-parallel) host path on CPU ranks (gloo).

The collectives of attention_relation_kl_b200.context_parallel (token
all-gather, statistics all-reduce, dX reduce-scatter) run for real between
2 and 3 gloo ranks; the two compute steps are replaced by an emulation that
evaluates the float64 oracle on a row partition of its own choosing, so that
what is tested here is the host logic: every rank must end with every row's
kl and the exact dX_s of its own tokens.  The kernels' own split of rows into
parts is tested on the GPU (tests/test_gpu_parts.py).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _owned_rows(N, part, n_parts):
    # the emulation's partition: blocks of 4 rows dealt round-robin
    return np.array([i for i in range(N) if (i // 4) % n_parts == part], dtype=np.int64)


def _emulated_fwd(pairs, causal, scale, part):
    from oracle import dense
    outs = []
    for xt, xs in pairs:
        B, H, N, _ = xt.shape
        kl = torch.zeros(B, H, N, dtype=torch.float32)
        st = torch.zeros(B, H, N, 4, dtype=torch.float32)
        rows = _owned_rows(N, *part)
        for b in range(B):
            for h in range(H):
                r = dense.fwd_rows(xt[b, h], xs[b, h], rows, causal)
                kl[b, h, rows] = torch.from_numpy(r["kl"]).float()
                st[b, h, rows] = torch.from_numpy(
                    np.stack([r["m"], r["lse_t"], r["lse_s"], r["w"]], axis=1)).float()
        outs.append((kl, st))
    return outs


def _emulated_bwd(pairs, stats, causal, scale, part):
    from oracle import dense
    dxs = []
    for (xt, xs), st in zip(pairs, stats):
        # the host must have combined every part's statistics by now
        assert torch.all(st[..., 1] != 0), "statistics of other parts' rows are missing"
        B, H, N, d = xt.shape
        dx = torch.zeros(B, H, N, d, dtype=torch.float32)
        rows = _owned_rows(N, *part)
        for b in range(B):
            for h in range(H):
                dx[b, h] = torch.from_numpy(dense.bwd_contrib(xt[b, h], xs[b, h], rows, None,
                                                              causal)).float()
        dxs.append(dx)
    return dxs


def _worker(rank, world, port, full_pairs, causal, out_kl, out_dx):
    import torch.distributed as dist
    from attention_relation_kl_b200.context_parallel import context_parallel_step
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = []
        for xt, xs in full_pairs:                    # [B, H, N, d] -> token-major shards
            n = xt.shape[2] // world
            tm = lambda x: x.permute(2, 0, 1, 3)[rank * n:(rank + 1) * n].contiguous()
            local.append((tm(xt), tm(xs)))
        kl, stats, dx_local = context_parallel_step(local, causal, fwd_part=_emulated_fwd,
                                                    bwd_part=_emulated_bwd)
        for r in range(len(full_pairs)):
            out_kl[r][rank].copy_(kl[r])
            out_dx[r][rank].copy_(dx_local[r])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (3, False)])
def test_context_parallel_host_path(world, causal):
    from oracle import dense
    import workload
    N = 24 * world
    pairs = []
    for seed in (3, 4):
        xt, xs = workload.gaussian_pair((1, 2, N, 8), seed=seed, noise=0.4, dtype=torch.float32)
        pairs.append((xt, xs))
    n = N // world
    out_kl = [torch.zeros(world, 1, 2, N).share_memory_() for _ in pairs]
    out_dx = [torch.zeros(world, n, 1, 2, 8).share_memory_() for _ in pairs]
    mp.spawn(_worker, args=(world, _free_port(), pairs, causal, out_kl, out_dx), nprocs=world,
             join=True)
    for r, (xt, xs) in enumerate(pairs):
        ref_kl = dense.fwd(xt, xs, causal)["kl"]
        ref_dx = dense.bwd(xt, xs, None, causal)                  # [1, 2, N, 8]
        for rank in range(world):
            np.testing.assert_allclose(out_kl[r][rank].numpy(), ref_kl, rtol=1e-5, atol=1e-7)
            want = ref_dx[:, :, rank * n:(rank + 1) * n].transpose(2, 0, 1, 3)
            np.testing.assert_allclose(out_dx[r][rank].numpy(), want, rtol=1e-4,
                                       atol=1e-6 * np.abs(ref_dx).max())


def test_single_process_is_the_plain_step():
    """Without a process group the step is one part of one: gather and
    reduce-scatter are identities."""
    from oracle import dense
    import workload
    from attention_relation_kl_b200.context_parallel import context_parallel_step
    xt, xs = workload.gaussian_pair((1, 1, 20, 8), seed=8, noise=0.3, dtype=torch.float32)
    local = [(xt.permute(2, 0, 1, 3).contiguous(), xs.permute(2, 0, 1, 3).contiguous())]
    kl, _, dx = context_parallel_step(local, True, fwd_part=_emulated_fwd, bwd_part=_emulated_bwd)
    np.testing.assert_allclose(kl[0].numpy(), dense.fwd(xt, xs)["kl"], rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(dx[0].numpy(), dense.bwd(xt, xs).transpose(2, 0, 1, 3), rtol=1e-4,
                               atol=1e-9)
