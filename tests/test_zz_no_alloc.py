"""relkl_fwd_noalloc: the forward for callers that cannot hand the library a
device workspace (for example a host framework that plans every device buffer
itself and gives a custom operation only its inputs and outputs).

The entry point takes no workspace and allocates nothing; its scratch is a
static device array inside librelkl.so.  This test calls it through the C ABI
twice in a row and checks both results against relkl_fwd (which uses a caller
workspace) within the parity tolerances the other tests use.  It lives in its
own file so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import attention_relation_kl_b200 as rk
import workload
from parity import assert_kl, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_noalloc_forward_matches_workspace_forward_twice():
    w = workload.tiny_custom(N=700, d=128, dtype="bf16", seed=41, B=1, H=3)
    xt, xs = workload.generate(w)["q"]
    gt, gs = xt.cuda(), xs.cuda()
    ref_kl, ref_st = rk.relkl_fwd(gt, gs)
    torch.cuda.synchronize()
    ref_kl, ref_st = to_np(ref_kl), to_np(ref_st)
    for _ in range(2):
        kl = torch.full((1, 3, 700), float("nan"), device="cuda")
        st = torch.full((1, 3, 700, 4), float("nan"), device="cuda")
        rk.relkl_fwd_noalloc(gt, gs, kl=kl, stats=st)
        torch.cuda.synchronize()
        got_kl, got_st = to_np(kl), to_np(st)
        assert np.isfinite(got_kl).all() and np.isfinite(got_st).all()
        assert_kl(got_kl, ref_kl, what="kl (no-alloc vs workspace forward)")
        np.testing.assert_allclose(got_st[..., :3], ref_st[..., :3], rtol=2e-5, atol=2e-5)
        w_err = np.abs(got_st[..., 3] - ref_st[..., 3])
        assert np.all(w_err <= 1e-3 * np.abs(ref_st[..., 3]) + 2e-5)
