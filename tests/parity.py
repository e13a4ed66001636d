"""Shared parity helpers: tolerances and oracle comparisons.

Tolerances (the relation-KL hot-path specification):
* per-row KL and the total loss: relative 1e-3; per row an absolute floor of
  1e-6 is added for rows whose exact KL is 0 or tiny (causal row 0, identical
  teacher and student);
* dX_s: max-norm relative 2e-2 for bf16 inputs with fp32 accumulation (the
  tensor-core path rounds G to bf16).  For the fp32 CUDA-core path the
  tolerance is derived for each test input by ``fp32_dx_tolerance`` from a
  rounding-error model of that path's arithmetic evaluated on the oracle's own
  R_t, R_s and X_s (no kernel output enters it);
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


U32 = 2.0 ** -24   # unit roundoff of float32


def fp32_dx_bound_unit(xt, xs, dkl=None, causal=True, scale=None, k_sigma=5.0):
    """Per-element bound on |dX_fp32 - dX| for one [n, d] unit, from the float32
    CUDA-core path's arithmetic applied to the oracle's R_t, R_s and X_s.

    Rounding errors are modelled as independent, zero-mean and uniform within
    half an ulp (standard deviation u/sqrt(3) of the rounded value, u = 2^-24),
    except where one rounded quantity is reused: a row's LSE enters every
    probability of that row, so its error adds coherently along the row.
      * logit z_ij = s S_ij,d with S_ij,k = sum_{m<=k} x_im x_jm (d fused
        multiply-adds, each rounding one partial sum, then the scale):
        sd(dz_ij)^2 = u^2 / 3 (s^2 sum_k S_ij,k^2 + z_ij^2), from the exact
        partial sums;
      * probability P_ij = expf(z_ij - lse_i) (expf within 2 ulp): independent
        relative error sd_ij^2 = sd(dz_ij)^2 + (u |z_ij - lse_i|)^2 / 3 + 4 u^2 / 3;
      * row LSE: error of its largest logit, of the exps it sums and of the
        sum's n_i roundings and the log: sd(dlse_i)^2 = max_j sd(dz_ij)^2
        + sum_j P_ij^2 sd_ij^2 + (n_i + lse_i^2) u^2 / 3;
      * G_ij = dkl_i (P_s - P_t)_ij, one more rounding: u |G_ij| / sqrt(3);
      * dX_rc = s sum_j (G_rj + G_jr) X_jc, accumulated over n terms:
        u sqrt(n / 3) s sum_j (|G_rj| + |G_jr|) |X_jc|.
    Row side: the LSE part is coherent, k_sigma sd(dlse_r) |sum_j P_rj X_jc|
    for teacher and student; everything else adds in quadrature.  Column side:
    the LSE of each row j is a separate quantity, so all terms add in
    quadrature.  Returns coherent part + k_sigma x quadrature part.  G + G^T
    has nearly cancelling rows (each row of G sums to zero), so the bound is
    set by the absolute sums rather than by |dX|: that ratio is the
    amplification the bound carries for this input.
    """
    from oracle import dense
    xt64, xs64 = dense.as_f64(xt), dense.as_f64(xs)
    n, d = xt64.shape
    s = 1.0 / np.sqrt(d) if not scale else float(scale)
    g_up = np.full(n, 1.0 / n) if dkl is None else np.asarray(dkl, np.float64).reshape(n)
    p_t, p_s = dense.relation_probs(xt64, xs64, causal, scale)
    ok = dense.allowed(np.arange(n), n, causal)
    n_row = ok.sum(axis=1).astype(np.float64)
    stats = dense.fwd_unit(xt64, xs64, causal, scale)
    u2 = U32 * U32
    sd = {}
    sd_lse = {}
    for name, x, p, lse in (("t", xt64, p_t, stats["lse_t"]), ("s", xs64, p_s, stats["lse_s"])):
        z = s * (x @ x.T)
        partial = np.cumsum(x[:, None, :] * x[None, :, :], axis=2)     # [n, n, d]
        sd_z2 = u2 / 3.0 * (s * s * (partial * partial).sum(axis=2) + z * z)
        del partial
        sd2 = np.where(ok, sd_z2 + u2 * (z - lse[:, None]) ** 2 / 3.0 + 4.0 * u2 / 3.0, 0.0)
        sd[name] = sd2
        sd_lse[name] = (np.where(ok, sd_z2, 0.0).max(axis=1) + (p * p * sd2).sum(axis=1)
                        + (n_row + lse * lse) * u2 / 3.0)
    G = g_up[:, None] * (p_s - p_t)
    ax = np.abs(xs64)
    x2 = xs64 * xs64
    # variance of dG from the independent per-entry errors, and of G's own rounding
    var_g = (g_up[:, None] ** 2) * (p_s * p_s * sd["s"] + p_t * p_t * sd["t"]) + u2 * G * G / 3.0
    # row side: independent part, and the coherent LSE part of row r
    var_row = var_g @ x2
    coh_row = k_sigma * np.abs(g_up)[:, None] * (np.sqrt(sd_lse["s"])[:, None] * np.abs(p_s @ xs64)
                                                  + np.sqrt(sd_lse["t"])[:, None] * np.abs(p_t @ xs64))
    # column side: row j's LSE error is independent of row j' != j
    var_lse_col = (g_up[:, None] ** 2) * (p_s * p_s * sd_lse["s"][:, None]
                                          + p_t * p_t * sd_lse["t"][:, None])
    var_col = (var_g + var_lse_col).T @ x2
    absG = np.abs(G)
    var_acc = (n / 3.0) * u2 * ((absG + absG.T) @ ax) ** 2
    return s * (coh_row + k_sigma * np.sqrt(var_row + var_col + var_acc))


def fp32_dx_tolerance(xt, xs, dkl=None, causal=True, scale=None, lengths=None):
    """Max-norm relative dX tolerance for the fp32 path on a [B, H, N, d] input:
    the largest per-element bound (fp32_dx_bound_unit) over every unit, divided
    by max |dX| over the whole tensor."""
    from oracle import dense
    xt64, xs64 = dense.as_f64(xt), dense.as_f64(xs)
    B, H, N, _ = xt64.shape
    g = None if dkl is None else dense.as_f64(dkl).reshape(B, H, N)
    ref = dense.bwd(xt64, xs64, g, causal, scale, lengths=lengths)
    worst = 0.0
    for b in range(B):
        L = N if lengths is None else max(0, min(N, int(lengths[b])))
        if L == 0:
            continue
        for h in range(H):
            bound = fp32_dx_bound_unit(xt64[b, h, :L], xs64[b, h, :L],
                                       None if g is None else g[b, h, :L], causal, scale)
            worst = max(worst, float(bound.max()))
    scale_ref = float(np.abs(ref).max())
    return worst / scale_ref if scale_ref > 0 else 1e-12
