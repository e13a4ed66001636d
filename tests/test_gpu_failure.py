"""Failure detection on the GPU without a fault: every device-side wait of the
tcgen05 kernels is bounded.  The test hook relkl_set_wait_timeout_ns(0) makes
the first wait that is not satisfied at once run out; the kernel records the
site in the workspace, every role leaves its loop, waits for its own copies and
MMAs in flight, frees TMEM and exits.  The host reads RELKL_ERR_TIMEOUT, and
the CUDA context stays usable: the next call with the normal bound is correct.
"""
import pytest
import torch

import attention_relation_kl_b200 as rk
import workload
from attention_relation_kl_b200 import _abi
from oracle import dense
from parity import DX_TOL_BF16, assert_dx, assert_kl, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _inputs():
    w = workload.tiny_custom(N=1024, d=128, dtype="bf16", seed=31, B=1, H=2)
    return workload.generate(w)["q"]


@pytest.mark.parametrize("phase", ["fwd", "bwd"])
def test_wait_timeout_is_reported_and_context_survives(phase):
    xt, xs = _inputs()
    gt, gs = xt.cuda(), xs.cuda()
    ws = torch.empty(rk.relkl_workspace_bytes(), dtype=torch.uint8, device="cuda")
    rk.relkl_workspace_init(ws)
    kl, st = rk.relkl_fwd(gt, gs, ws=ws)
    torch.cuda.synchronize()
    assert rk.relkl_get_device_error(ws)[0] == _abi.RELKL_OK
    old = rk.relkl_set_wait_timeout_ns(0)
    try:
        if phase == "fwd":
            rk.relkl_fwd(gt, gs, ws=ws)
        else:
            rk.relkl_bwd(gt, gs, st, ws=ws)
        code, where = rk.relkl_get_device_error(ws)
    finally:
        rk.relkl_set_wait_timeout_ns(old)
    assert code == _abi.RELKL_ERR_TIMEOUT and where != 0
    # the record sticks until cleared
    assert rk.relkl_get_device_error(ws)[0] == _abi.RELKL_ERR_TIMEOUT
    rk.relkl_workspace_init(ws)
    kl, st = rk.relkl_fwd(gt, gs, ws=ws)
    dx = rk.relkl_bwd(gt, gs, st, ws=ws)
    torch.cuda.synchronize()
    assert rk.relkl_get_device_error(ws)[0] == _abi.RELKL_OK
    assert_kl(to_np(kl), dense.fwd(xt, xs)["kl"])
    assert_dx(to_np(dx), dense.bwd(xt, xs), DX_TOL_BF16)
