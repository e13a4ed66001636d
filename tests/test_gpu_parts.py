"""GPU: one problem split into parts (relkl_fwd_qkv_part / relkl_bwd_qkv_part).

The parts that the ranks of a row-sharded (context-parallel) run would take
are run one after the other on one GPU: every row's kl and statistics must be
written by exactly one part, bit for bit as the single call writes them, and
the parts' dX_s contributions must add up to the single call's dX_s and to the
float64 oracle's.  Every kernel family: the one-block (N <= 4096) and
paired-block (N > 4096) backwards at d = 128, d = 64 and the CUDA-core fp32
path; both masks.
"""
import numpy as np
import pytest
import torch

import attention_relation_kl_b200 as rk
import workload
from oracle import dense
from parity import DX_TOL_BF16, assert_dx, assert_kl, fp32_dx_tolerance, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("N,d,dtype,causal,n_parts", [
    (700, 128, "bf16", True, 3),
    (4480, 128, "bf16", True, 4),      # paired-block backward, 35 row blocks
    (4200, 128, "bf16", False, 5),
    (513, 64, "bf16", True, 2),
    (150, 64, "fp32", False, 3),
    (300, 128, "bf16", True, 7),       # more parts than some units' work items
])
def test_parts_add_up_to_the_whole(N, d, dtype, causal, n_parts):
    w = workload.tiny_custom(N=N, d=d, dtype=dtype, seed=N + n_parts, causal=causal, B=2, H=1)
    xt, xs = workload.generate(w)["q"]
    gt, gs = xt.cuda(), xs.cuda()
    kl_full, st_full = rk.relkl_fwd(gt, gs, causal)
    dx_full = rk.relkl_bwd(gt, gs, st_full, None, causal)
    kl_sum = torch.zeros_like(kl_full)
    st_sum = torch.zeros_like(st_full)
    written = torch.zeros(kl_full.shape, dtype=torch.int32, device="cuda")
    parts = []
    for p in range(n_parts):
        (kl, st), = rk.relkl_fwd_qkv([(gt, gs)], causal, part=(p, n_parts))
        kl_sum += kl
        st_sum += st
        written += (st != 0).any(dim=-1).int()
        parts.append(st)
    torch.cuda.synchronize()
    assert torch.all(written == 1), "every row belongs to exactly one part"
    assert torch.equal(kl_sum, kl_full) and torch.equal(st_sum, st_full)
    dx_sum = torch.zeros_like(dx_full)
    for p in range(n_parts):
        dx_sum += rk.relkl_bwd_qkv([(gt, gs)], [st_full], None, causal, part=(p, n_parts))[0]
    torch.cuda.synchronize()
    code, where = rk.relkl_get_device_error()
    assert code == 0, f"device wait ran out at site {where}"
    # the sum of the parts is the single call up to the order of fp32 additions
    assert_dx(to_np(dx_sum), to_np(dx_full), 1e-5)
    tol = DX_TOL_BF16 if dtype == "bf16" else fp32_dx_tolerance(xt, xs, None, causal)
    assert_dx(to_np(dx_sum), dense.bwd(xt, xs, None, causal), tol)
    assert_kl(to_np(kl_sum), dense.fwd(xt, xs, causal)["kl"])


def test_context_parallel_step_on_one_rank_is_the_plain_call():
    from attention_relation_kl_b200.context_parallel import context_parallel_step
    w = workload.Workload("cp1", B=1, H=2, H_kv=1, N=1024, d=128, dtype="bf16", causal=True,
                          relations=("q", "k", "v"), rope_base=1e4, pi_factor=8.0, v_noise=0.1,
                          seed=57)
    x = workload.generate(w)
    local = [(x[r][0].cuda().permute(2, 0, 1, 3).contiguous(),
              x[r][1].cuda().permute(2, 0, 1, 3).contiguous()) for r in w.relations]
    kl, stats, dx_local = context_parallel_step(local, True)
    torch.cuda.synchronize()
    for i, r in enumerate(w.relations):
        assert_kl(to_np(kl[i]), dense.fwd(*x[r])["kl"], what=f"kl[{r}]")
        ref = dense.bwd(*x[r])                               # [B, H, N, d]
        assert_dx(to_np(dx_local[i]).transpose(1, 2, 0, 3), ref, DX_TOL_BF16)
