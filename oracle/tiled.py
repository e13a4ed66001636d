"""Float64 tiled (linear-memory) restatements of the relation-KL computation.

TEST INFRASTRUCTURE.  Only the tests may import this module; it shares no code
with the CUDA path.

The pages claim the linear-memory kernel is *exact*: it reaches the same KL
and gradients as the materialised computation while keeping only O(n) row
statistics (LinearARD abstract on the mlsanity.com index page; pith.science
verdict, ``pith_extraction.key_machinery`` and the desk editor's letter, which
cite Propositions 3.2/3.3 and Table 8).  The functions here restate the tiled
algorithms in plain float64 so that a test can hold them against the dense
definition in ``oracle.dense`` to ~1e-12; no N x N array is ever formed here.

``two_phase``   the pages' scheme (``key_machinery``): Phase 1 stores only the
                per-row LSE of teacher and student, built by an online
                max-and-rescale sweep over column tiles; Phase 2 recomputes the
                masked logit tiles, rebuilds R_t and R_s from the stored LSEs,
                accumulates the KL and forms the gradient tile
                G = dkl * (R_s - R_t), streaming G X_s into the row block and
                G^T X_s into the column block.

``one_pass_shared_max``  the forward formulation the GPU kernels use: one
                online sweep with a single running maximum m shared by teacher
                and student, accumulating S_t = sum e^(z_t - m),
                C = sum (e^(z_s - m) - e^(z_t - m)) and A = sum e^(z_t - m)(z_t - z_s).
                Then lse_t = m + ln S_t, lse_s = m + ln(S_t + C), w = A / S_t and
                kl = w + log1p(C / S_t).  This is kl = w + lse_s - lse_t
                rearranged so that the difference lse_s - lse_t is never formed
                from two large numbers.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

from .dense import as_f64

__all__ = ["two_phase", "one_pass_shared_max"]


def _tile_mask(i0, i1, j0, j1, causal):
    rows = np.arange(i0, i1)[:, None]
    cols = np.arange(j0, j1)[None, :]
    return cols <= rows if causal else np.ones((i1 - i0, j1 - j0), dtype=bool)


def _col_range(i1, N, causal):
    return i1 if causal else N


def two_phase(xt, xs, dkl=None, causal: bool = True, scale: Optional[float] = None,
              tile_m: int = 64, tile_n: int = 64) -> Dict[str, np.ndarray]:
    """Pages' two-phase tiled algorithm.  Returns lse_t, lse_s, kl and dx_s."""
    xt, xs = as_f64(xt), as_f64(xs)
    N, d = xt.shape
    s = 1.0 / np.sqrt(d) if not scale else float(scale)
    g_up = np.full(N, 1.0 / N) if dkl is None else as_f64(dkl).reshape(N)

    # Phase 1: per-row log-sum-exp, online over column tiles.
    lse = {}
    for name, x in (("t", xt), ("s", xs)):
        out = np.empty(N)
        for i0 in range(0, N, tile_m):
            i1 = min(N, i0 + tile_m)
            run_max = np.full(i1 - i0, -np.inf)
            run_sum = np.zeros(i1 - i0)
            for j0 in range(0, _col_range(i1, N, causal), tile_n):
                j1 = min(N, j0 + tile_n)
                ok = _tile_mask(i0, i1, j0, j1, causal)
                z = np.where(ok, s * (x[i0:i1] @ x[j0:j1].T), -np.inf)
                new_max = np.maximum(run_max, z.max(axis=1))
                # rows whose tile is fully masked keep their state
                safe = np.where(np.isfinite(new_max), new_max, 0.0)
                run_sum = run_sum * np.exp(run_max - safe) + np.exp(z - safe[:, None]).sum(axis=1)
                run_max = new_max
            out[i0:i1] = run_max + np.log(run_sum)
        lse[name] = out

    # Phase 2: recompute tiles, rebuild R_t and R_s, accumulate KL and gradient.
    kl = np.zeros(N)
    dx = np.zeros_like(xs)
    for i0 in range(0, N, tile_m):
        i1 = min(N, i0 + tile_m)
        for j0 in range(0, _col_range(i1, N, causal), tile_n):
            j1 = min(N, j0 + tile_n)
            ok = _tile_mask(i0, i1, j0, j1, causal)
            if not ok.any():
                continue
            zt = s * (xt[i0:i1] @ xt[j0:j1].T)
            zs = s * (xs[i0:i1] @ xs[j0:j1].T)
            log_rt = zt - lse["t"][i0:i1, None]
            log_rs = zs - lse["s"][i0:i1, None]
            rt = np.where(ok, np.exp(log_rt), 0.0)
            rs = np.where(ok, np.exp(log_rs), 0.0)
            kl[i0:i1] += (rt * np.where(ok, log_rt - log_rs, 0.0)).sum(axis=1)
            g = g_up[i0:i1, None] * (rs - rt)
            dx[i0:i1] += s * (g @ xs[j0:j1])
            dx[j0:j1] += s * (g.T @ xs[i0:i1])
    return {"lse_t": lse["t"], "lse_s": lse["s"], "kl": kl, "dx": dx}


def one_pass_shared_max(xt, xs, causal: bool = True, scale: Optional[float] = None,
                        tile_m: int = 64, tile_n: int = 64) -> Dict[str, np.ndarray]:
    """Forward statistics by the shared-max one-pass sweep (see module doc)."""
    xt, xs = as_f64(xt), as_f64(xs)
    N, d = xt.shape
    s = 1.0 / np.sqrt(d) if not scale else float(scale)
    res = {k: np.empty(N) for k in ("kl", "lse_t", "lse_s", "w", "m")}
    for i0 in range(0, N, tile_m):
        i1 = min(N, i0 + tile_m)
        m = np.full(i1 - i0, -np.inf)
        S_t = np.zeros(i1 - i0)
        C = np.zeros(i1 - i0)
        A = np.zeros(i1 - i0)
        for j0 in range(0, _col_range(i1, N, causal), tile_n):
            j1 = min(N, j0 + tile_n)
            ok = _tile_mask(i0, i1, j0, j1, causal)
            zt = s * (xt[i0:i1] @ xt[j0:j1].T)
            zs = s * (xs[i0:i1] @ xs[j0:j1].T)
            tile_max = np.where(ok, np.maximum(zt, zs), -np.inf).max(axis=1)
            m_new = np.maximum(m, tile_max)
            safe = np.where(np.isfinite(m_new), m_new, 0.0)
            alpha = np.exp(m - safe)                      # 0 when m was -inf
            e_t = np.where(ok, np.exp(zt - safe[:, None]), 0.0)
            e_s = np.where(ok, np.exp(zs - safe[:, None]), 0.0)
            S_t = S_t * alpha + e_t.sum(axis=1)
            C = C * alpha + (e_s - e_t).sum(axis=1)
            A = A * alpha + (e_t * np.where(ok, zt - zs, 0.0)).sum(axis=1)
            m = m_new
        res["m"][i0:i1] = m
        res["lse_t"][i0:i1] = m + np.log(S_t)
        res["lse_s"][i0:i1] = m + np.log(S_t + C)
        res["w"][i0:i1] = A / S_t
        res["kl"][i0:i1] = A / S_t + np.log1p(C / S_t)
    return res
