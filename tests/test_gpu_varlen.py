"""GPU parity for packed variable-length sequences (relkl_desc.cu_seqlens).

Sequences of unequal lengths (empty ones included) lie back to back on one
token axis, followed by tokens that belong to no sequence and hold large
garbage values.  Each (sequence, head) must equal the float64 oracle of that
sequence alone, on every kernel family (one-block and paired-block backwards
at d = 128, d = 64, the CUDA-core fp32 path) and both masks; the tokens past
the last sequence must keep kl = 0 and get dX_s = 0.
"""
import numpy as np
import pytest
import torch

import attention_relation_kl_b200 as rk
import workload
from oracle import dense
from parity import DX_TOL_BF16, assert_dx, assert_kl, assert_stats, fp32_dx_tolerance, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _packed(lens, H, d, dtype, seed, tail=11):
    total = sum(lens) + tail
    w = workload.tiny_custom(N=total, d=d, dtype=dtype, seed=seed, pi_factor=4.0, B=1, H=H)
    xt, xs = workload.generate(w)["q"]
    xt, xs = xt.clone(), xs.clone()
    xt[:, :, total - tail:] = 30.0            # tokens of no sequence: must not leak
    xs[:, :, total - tail:] = -45.0
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return xt, xs, cu, total - tail


@pytest.mark.parametrize("lens,d,dtype,causal", [
    ([300, 0, 1, 129, 700, 57], 128, "bf16", True),
    ([300, 0, 1, 129, 700, 57], 128, "bf16", False),
    ([4300, 200, 4097, 5], 128, "bf16", True),        # paired-block backward
    ([4300, 200, 4097, 5], 128, "bf16", False),
    ([513, 64, 1000], 64, "bf16", True),
    ([150, 33, 0, 97], 64, "fp32", False),
])
def test_packed_sequences(lens, d, dtype, causal):
    H = 2
    xt, xs, cu, end = _packed(lens, H, d, dtype, seed=sum(lens) + d)
    gt, gs = xt.cuda(), xs.cuda()
    gcu = torch.from_numpy(cu).cuda()
    ms = max(lens)
    kl, st = rk.relkl_fwd(gt, gs, causal, cu_seqlens=gcu, max_seqlen=ms)
    dx = rk.relkl_bwd(gt, gs, st, None, causal, cu_seqlens=gcu, max_seqlen=ms)
    torch.cuda.synchronize()
    code, where = rk.relkl_get_device_error()
    assert code == 0, f"device wait ran out at site {where}"
    ref = dense.fwd_varlen(xt, xs, cu, causal)
    assert_kl(to_np(kl), ref["kl"])
    assert_stats(to_np(st)[:, :, :end], {k: v[:, :, :end] for k, v in ref.items()})
    assert np.all(to_np(kl)[:, :, end:] == 0) and np.all(to_np(st)[:, :, end:] == 0)
    ref_dx = dense.bwd_varlen(xt, xs, cu, None, causal)
    tol = DX_TOL_BF16 if dtype == "bf16" else max(
        fp32_dx_tolerance(xt[:, :, a:b], xs[:, :, a:b], None, causal)
        for a, b in zip(cu[:-1], cu[1:]) if b > a)
    assert_dx(to_np(dx), ref_dx, tol)
    assert np.all(to_np(dx)[:, :, end:] == 0)
    # a sequence of one token: its only row has R_t = R_s = 1, so its gradient is exactly 0
    for a, b in zip(cu[:-1], cu[1:]):
        if b - a == 1:
            assert np.all(to_np(dx)[:, :, a] == 0)


def test_packed_sequences_fused_qkv_and_upstream_gradient():
    lens = [700, 260, 1]
    H, H_kv, d = 4, 2, 128
    total = sum(lens)
    g = workload.Workload("packed_qkv", B=1, H=H, H_kv=H_kv, N=total, d=d, dtype="bf16",
                          causal=True, relations=("q", "k", "v"), rope_base=5e5, pi_factor=4.0,
                          v_noise=0.05, seed=71)
    x = workload.generate(g)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    gcu = torch.from_numpy(cu).cuda()
    pairs = [(x[r][0].cuda(), x[r][1].cuda()) for r in "qkv"]
    dkl = {r: torch.randn(1, g.heads(r), total, generator=torch.Generator().manual_seed(5)) / 300
           for r in "qkv"}
    outs = rk.relkl_fwd_qkv(pairs, cu_seqlens=gcu, max_seqlen=max(lens))
    dxs = rk.relkl_bwd_qkv(pairs, [o[1] for o in outs], [dkl[r].cuda() for r in "qkv"],
                           cu_seqlens=gcu, max_seqlen=max(lens))
    torch.cuda.synchronize()
    for r, (kl, _), dx in zip("qkv", outs, dxs):
        assert_kl(to_np(kl), dense.fwd_varlen(*x[r], cu)["kl"], what=f"kl[{r}]")
        assert_dx(to_np(dx), dense.bwd_varlen(*x[r], cu, dkl[r]), DX_TOL_BF16)
