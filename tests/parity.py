"""Shared parity helpers: tolerances and oracle comparisons.

Tolerances (the relation-KL hot-path specification):
* per-row KL and the total loss: relative 1e-3; per row an absolute floor of
  1e-6 is added for rows whose exact KL is 0 or tiny (causal row 0, identical
  teacher and student);
* dX_s: max-norm relative 2e-2 for bf16 inputs with fp32 accumulation (the
  tensor-core path rounds G to bf16); 2e-4 for the fp32 CUDA-core path.  The
  fp32 bound: logits of size |z| <~ 12 carry ~1e-6 absolute error, so each
  probability carries ~2e-6 relative error; G is a difference of nearly equal
  probabilities and dX = s (G + G^T) X cancels (every row of G sums to zero),
  which amplifies the error by sum|G||x| / |sum G x|, observed up to ~40 on
  these inputs: 2e-6 * 40 * 2 (margin) ~ 2e-4;
* statistics: lse and m to 2e-5 relative + 2e-5 absolute (fp32 logits of
  magnitude ~10), w like kl.
"""
import numpy as np
import torch

KL_RTOL, KL_ATOL = 1e-3, 1e-6
DX_TOL_BF16, DX_TOL_FP32 = 2e-2, 2e-4


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_kl(got, ref, what="kl"):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    bad = err > KL_RTOL * np.abs(ref) + KL_ATOL
    assert not bad.any(), (f"{what}: {bad.sum()} rows out of tolerance; worst at "
                           f"{np.unravel_index(np.argmax(err - KL_RTOL * np.abs(ref)), err.shape)}: "
                           f"got {got.flat[np.argmax(err - KL_RTOL * np.abs(ref))]!r} "
                           f"ref {ref.flat[np.argmax(err - KL_RTOL * np.abs(ref))]!r}")
    tot_g, tot_r = got.sum(), ref.sum()
    assert abs(tot_g - tot_r) <= KL_RTOL * abs(tot_r) + KL_ATOL, (what, tot_g, tot_r)


def assert_stats(got_stats, ref, rows=None):
    """got_stats [..., 4] = (m, lse_t, lse_s, w) against the oracle's dict."""
    g = np.asarray(got_stats, np.float64)
    for k, name in ((0, "m"), (1, "lse_t"), (2, "lse_s")):
        r = np.asarray(ref[name], np.float64)
        np.testing.assert_allclose(g[..., k], r, rtol=2e-5, atol=2e-5, err_msg=name)
    w_err = np.abs(g[..., 3] - ref["w"])
    assert np.all(w_err <= 1e-3 * np.abs(ref["w"]) + 2e-5), ("w", w_err.max())


def assert_dx(got, ref, tol):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    scale = np.max(np.abs(ref))
    err = np.max(np.abs(got - ref))
    if scale == 0.0:
        assert err <= 1e-12, err
    else:
        assert err <= tol * scale, f"dX max-norm relative error {err / scale:.3e} > {tol}"
