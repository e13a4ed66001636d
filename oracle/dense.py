"""Float64 CPU oracle for the relation-KL distillation loss and its gradient.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference arm may import this module.  It shares no code
with the CUDA path and is never called by the product.

What it computes (LinearARD, arXiv 2604.00004; the definitions are in the
pith.science verdict page, field ``pith_extraction.key_machinery``, repeated in
``core_discovery``; the abstract on the mlsanity.com index page names the
Q/Q, K/K and V/V relations and the forward KL):

* relation logits of one (batch, head, X) unit, for m in {teacher, student}:
      Z_m = X_m X_m^T / sqrt(d) + M
  with M the additive mask: 0 where column j is allowed for row i, -inf where
  it is not.  The pages name M without defining it; the reading taken here is
  the causal mask j <= i (a token relates to itself); ``causal=False`` gives
  full rows.
* row distributions R_m(i, :) = softmax(Z_m(i, :)), with the per-row
  log-sum-exp LSE_m(i) = log sum_k exp Z_m(i, k);
* the per-row forward KL with the teacher as target,
      kl_i = D_KL(R_t(i,:) || R_s(i,:)) = sum_j R_t(i,j) (log R_t(i,j) - log R_s(i,j)),
  and the loss L = (1/n) sum_i kl_i;
* the gradient identity dL/dZ_s(i,j) = (R_s(i,j) - R_t(i,j)) / n.  With an
  upstream gradient dkl_i per row (1/n for L) the logit gradient is
  G(i,j) = dkl_i (R_s(i,j) - R_t(i,j)) on allowed entries, 0 elsewhere.  Since
  Z_s = X_s X_s^T / sqrt(d) uses X_s on both sides, the chain rule gives
      dX_s = (G + G^T) X_s / sqrt(d).
  The pages stop before writing this step (the ``key_machinery`` text is cut
  off); it is the plain chain rule, and the teacher gets no gradient (frozen).

Besides kl the oracle returns the O(n) row statistics the pages' kernel keeps:
lse_t, lse_s, the weighted term w_i = sum_j R_t(i,j) (Z_t - Z_s)(i,j) (so that
kl_i = w_i + lse_s(i) - lse_t(i)) and the shared row maximum
m_i = max_j max(Z_t(i,j), Z_s(i,j)).

Everything is float64 NumPy: the inputs are converted exactly (bf16 and fp32
values are representable in float64).  For large N the same per-row arithmetic
runs over slabs of rows so that no N x N matrix is held; a test checks that the
slabbed and the one-slab results agree.
"""
from __future__ import annotations

from typing import Dict, Iterable, Optional

import numpy as np
import torch

__all__ = ["as_f64", "relation_logits", "allowed", "fwd_unit", "bwd_unit",
           "fwd_rows", "bwd_rows", "fwd", "bwd", "unit_loss", "relation_probs", "bwd_contrib",
           "fwd_varlen", "bwd_varlen"]


def as_f64(x) -> np.ndarray:
    """Exact float64 copy of a NumPy array or a (CPU) torch tensor."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if x.dtype in (torch.bfloat16, torch.float16):   # no NumPy type: widen exactly first
            x = x.float()
        x = x.numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _scale(d: int, scale: Optional[float]) -> float:
    return 1.0 / np.sqrt(d) if not scale else float(scale)


def relation_logits(x_rows: np.ndarray, x_all: np.ndarray, scale: float) -> np.ndarray:
    """Z(rows, :) = X[rows] X^T * scale (unmasked)."""
    return scale * (x_rows @ x_all.T)


def allowed(rows: np.ndarray, n_cols: int, causal: bool) -> np.ndarray:
    """Boolean mask of allowed (i, j): j <= i when causal, everything otherwise."""
    cols = np.arange(n_cols)
    if causal:
        return cols[None, :] <= rows[:, None]
    return np.ones((rows.shape[0], n_cols), dtype=bool)


def _masked_log_softmax(z: np.ndarray, ok: np.ndarray):
    zm = np.where(ok, z, -np.inf)
    mx = zm.max(axis=1)
    lse = mx + np.log(np.exp(zm - mx[:, None]).sum(axis=1))
    return zm - lse[:, None], lse, mx


def _row_stats(zt: np.ndarray, zs: np.ndarray, ok: np.ndarray) -> Dict[str, np.ndarray]:
    logp_t, lse_t, mx_t = _masked_log_softmax(zt, ok)
    logp_s, lse_s, mx_s = _masked_log_softmax(zs, ok)
    p_t = np.where(ok, np.exp(logp_t), 0.0)
    with np.errstate(invalid="ignore"):          # -inf - -inf on masked entries
        diff_logp = np.where(ok, logp_t - logp_s, 0.0)
    kl = (p_t * diff_logp).sum(axis=1)
    w = (p_t * np.where(ok, zt - zs, 0.0)).sum(axis=1)
    return {"kl": kl, "lse_t": lse_t, "lse_s": lse_s, "w": w, "m": np.maximum(mx_t, mx_s)}


def fwd_rows(xt, xs, rows: Iterable[int], causal: bool = True,
             scale: Optional[float] = None) -> Dict[str, np.ndarray]:
    """Row statistics (kl, lse_t, lse_s, w, m) of the selected rows of one unit."""
    xt, xs = as_f64(xt), as_f64(xs)
    rows = np.asarray(list(rows), dtype=np.int64)
    N, d = xt.shape
    s = _scale(d, scale)
    ncol = int(rows.max()) + 1 if (causal and rows.size) else N
    zt = relation_logits(xt[rows], xt[:ncol], s)
    zs = relation_logits(xs[rows], xs[:ncol], s)
    return _row_stats(zt, zs, allowed(rows, ncol, causal))


def fwd_unit(xt, xs, causal: bool = True, scale: Optional[float] = None,
             slab: int = 2048) -> Dict[str, np.ndarray]:
    """Row statistics of every row of one unit ([N, d] teacher and student)."""
    xt, xs = as_f64(xt), as_f64(xs)
    N = xt.shape[0]
    parts = [fwd_rows(xt, xs, range(r0, min(N, r0 + slab)), causal, scale)
             for r0 in range(0, N, slab)]
    return {k: np.concatenate([p[k] for p in parts]) for k in parts[0]}


def _default_dkl(dkl, N: int) -> np.ndarray:
    if dkl is None:
        return np.full(N, 1.0 / N)
    return as_f64(dkl).reshape(N)


def bwd_unit(xt, xs, dkl=None, causal: bool = True, scale: Optional[float] = None,
             slab: int = 2048) -> np.ndarray:
    """dL/dX_s of one unit, L = sum_i dkl_i kl_i (dkl defaults to 1/N: the mean KL)."""
    xt, xs = as_f64(xt), as_f64(xs)
    N, d = xt.shape
    s = _scale(d, scale)
    g_up = _default_dkl(dkl, N)
    dx = np.zeros_like(xs)
    for r0 in range(0, N, slab):
        rows = np.arange(r0, min(N, r0 + slab))
        ncol = int(rows[-1]) + 1 if causal else N
        ok = allowed(rows, ncol, causal)
        logp_t, _, _ = _masked_log_softmax(relation_logits(xt[rows], xt[:ncol], s), ok)
        logp_s, _, _ = _masked_log_softmax(relation_logits(xs[rows], xs[:ncol], s), ok)
        g = g_up[rows, None] * np.where(ok, np.exp(logp_s) - np.exp(logp_t), 0.0)
        dx[rows] += s * (g @ xs[:ncol])          # G X_s   (row side)
        dx[:ncol] += s * (g.T @ xs[rows])        # G^T X_s (column side)
    return dx


def bwd_rows(xt, xs, rows: Iterable[int], dkl=None, causal: bool = True,
             scale: Optional[float] = None, slab: int = 2048,
             lse: Optional[Dict[str, np.ndarray]] = None) -> np.ndarray:
    """Selected rows of dL/dX_s for one unit.

    Row r of (G + G^T) X_s needs row r of G (from row r's LSEs) and column r of
    G, which involves the LSEs of every row j that may attend to r.  Those come
    from ``fwd_unit`` (or are passed in as ``lse``, a dict holding the oracle's
    own ``lse_t`` and ``lse_s``).
    """
    xt, xs = as_f64(xt), as_f64(xs)
    rows = np.asarray(list(rows), dtype=np.int64)
    N, d = xt.shape
    s = _scale(d, scale)
    g_up = _default_dkl(dkl, N)
    if lse is None:
        lse = fwd_unit(xt, xs, causal, scale, slab)
    lse_t, lse_s = np.asarray(lse["lse_t"]), np.asarray(lse["lse_s"])
    # row side: G(r, j) for allowed j
    ok_r = allowed(rows, N, causal)
    zt_r = relation_logits(xt[rows], xt, s)
    zs_r = relation_logits(xs[rows], xs, s)
    with np.errstate(over="ignore"):             # masked entries may overflow; dropped
        g_row = g_up[rows, None] * np.where(
            ok_r, np.exp(zs_r - lse_s[rows, None]) - np.exp(zt_r - lse_t[rows, None]), 0.0)
    # column side: G(j, r) for every row j that may attend to column r
    if causal:                                                       # [N, R]: j >= r
        ok_c = np.arange(N)[:, None] >= rows[None, :]
    else:
        ok_c = np.ones((N, rows.size), dtype=bool)
    zt_c = relation_logits(xt, xt[rows], s)                           # [N, R]
    zs_c = relation_logits(xs, xs[rows], s)
    with np.errstate(over="ignore"):
        g_col = g_up[:, None] * np.where(
            ok_c, np.exp(zs_c - lse_s[:, None]) - np.exp(zt_c - lse_t[:, None]), 0.0)
    return s * (g_row @ xs + g_col.T @ xs)


def _valid_len(lengths, b: int, N: int) -> int:
    """Right padding: batch element b holds lengths[b] real tokens (clamped to
    [0, N]); the rest are padding, excluded from every row distribution."""
    return N if lengths is None else max(0, min(N, int(np.asarray(lengths)[b])))


def fwd(xt, xs, causal: bool = True, scale: Optional[float] = None,
        slab: int = 2048, lengths=None) -> Dict[str, np.ndarray]:
    """Batched forward over [B, H, N, d]; each statistic comes back as [B, H, N].

    With ``lengths`` ([B]), batch element b is the sequence of its first
    lengths[b] tokens; its padding rows come back as 0.
    """
    xt, xs = as_f64(xt), as_f64(xs)
    B, H, N, _ = xt.shape
    out = {k: np.zeros((B, H, N)) for k in ("kl", "lse_t", "lse_s", "w", "m")}
    for b in range(B):
        L = _valid_len(lengths, b, N)
        if L == 0:
            continue
        for h in range(H):
            r = fwd_unit(xt[b, h, :L], xs[b, h, :L], causal, scale, slab)
            for k in out:
                out[k][b, h, :L] = r[k]
    return out


def bwd(xt, xs, dkl=None, causal: bool = True, scale: Optional[float] = None,
        slab: int = 2048, lengths=None) -> np.ndarray:
    """Batched backward over [B, H, N, d]; ``dkl`` is [B, H, N] or None (1/n per
    row, n the sequence length: N, or lengths[b] with padding, whose rows get 0)."""
    xt, xs = as_f64(xt), as_f64(xs)
    B, H, N, _ = xt.shape
    g = None if dkl is None else as_f64(dkl).reshape(B, H, N)
    dx = np.zeros_like(xs)
    for b in range(B):
        L = _valid_len(lengths, b, N)
        if L == 0:
            continue
        for h in range(H):
            dx[b, h, :L] = bwd_unit(xt[b, h, :L], xs[b, h, :L],
                                    None if g is None else g[b, h, :L], causal, scale, slab)
    return dx


def unit_loss(kl_rows: np.ndarray) -> float:
    """L = (1/n) sum_i kl_i for one unit's rows."""
    kl_rows = np.asarray(kl_rows, dtype=np.float64)
    return float(kl_rows.sum() / kl_rows.shape[-1])


def relation_probs(xt, xs, causal: bool = True, scale: Optional[float] = None):
    """Dense row distributions (R_t, R_s) of one small unit, zero on masked
    entries.  For tests that need the whole matrices (e.g. rounding-error
    bounds); the product path never forms them."""
    xt, xs = as_f64(xt), as_f64(xs)
    N, d = xt.shape
    s = _scale(d, scale)
    ok = allowed(np.arange(N), N, causal)
    logp_t, _, _ = _masked_log_softmax(relation_logits(xt, xt, s), ok)
    logp_s, _, _ = _masked_log_softmax(relation_logits(xs, xs, s), ok)
    return np.where(ok, np.exp(logp_t), 0.0), np.where(ok, np.exp(logp_s), 0.0)


def bwd_contrib(xt, xs, rows: Iterable[int], dkl=None, causal: bool = True,
                scale: Optional[float] = None) -> np.ndarray:
    """The share of dL/dX_s that the given rows of G produce.

    dX_s = s (G + G^T) X_s is linear in G, and G's rows are formed
    independently (row i needs only row i's logits and LSEs), so dX_s is the
    sum over rows i of s (e_i G(i,:) X_s + G(i,:)^T X_s[i]): the first term
    lands on row i, the second on every column row j that row i sees.  This
    returns that sum over ``rows`` only; summing it over a partition of the
    rows gives ``bwd_unit``.
    """
    xt, xs = as_f64(xt), as_f64(xs)
    rows = np.asarray(list(rows), dtype=np.int64)
    N, d = xt.shape
    s = _scale(d, scale)
    g_up = _default_dkl(dkl, N)
    dx = np.zeros_like(xs)
    if rows.size == 0:
        return dx
    ok = allowed(rows, N, causal)
    logp_t, _, _ = _masked_log_softmax(relation_logits(xt[rows], xt, s), ok)
    logp_s, _, _ = _masked_log_softmax(relation_logits(xs[rows], xs, s), ok)
    g = g_up[rows, None] * np.where(ok, np.exp(logp_s) - np.exp(logp_t), 0.0)
    dx[rows] += s * (g @ xs)              # row side
    dx += s * (g.T @ xs[rows])            # column side
    return dx


def _seq_bounds(cu_seqlens, N: int):
    cu = np.asarray(cu_seqlens, dtype=np.int64).reshape(-1)
    if cu.size < 1 or cu[0] != 0 or np.any(np.diff(cu) < 0) or cu[-1] > N:
        raise ValueError("cu_seqlens must start at 0, not decrease and end at most at N")
    return cu


def fwd_varlen(xt, xs, cu_seqlens, causal: bool = True, scale: Optional[float] = None,
               slab: int = 2048) -> Dict[str, np.ndarray]:
    """Packed variable-length sequences: [1, H, N, d] holds sequences back to
    back on one token axis, sequence k on tokens [cu[k], cu[k+1]).  Each
    sequence is its own relation: its rows see only its own tokens (masked as
    usual inside it).  Statistics come back as [1, H, N]; tokens past the last
    sequence stay 0."""
    xt, xs = as_f64(xt), as_f64(xs)
    _, H, N, _ = xt.shape
    cu = _seq_bounds(cu_seqlens, N)
    out = {k: np.zeros((1, H, N)) for k in ("kl", "lse_t", "lse_s", "w", "m")}
    for a, b in zip(cu[:-1], cu[1:]):
        if b == a:
            continue
        for h in range(H):
            r = fwd_unit(xt[0, h, a:b], xs[0, h, a:b], causal, scale, slab)
            for k in out:
                out[k][0, h, a:b] = r[k]
    return out


def bwd_varlen(xt, xs, cu_seqlens, dkl=None, causal: bool = True,
               scale: Optional[float] = None, slab: int = 2048) -> np.ndarray:
    """dL/dX_s of packed sequences; ``dkl`` is [1, H, N] or None (1/L_k on every
    row of a sequence of length L_k).  Tokens past the last sequence get 0."""
    xt, xs = as_f64(xt), as_f64(xs)
    _, H, N, _ = xt.shape
    cu = _seq_bounds(cu_seqlens, N)
    g = None if dkl is None else as_f64(dkl).reshape(1, H, N)
    dx = np.zeros_like(xs)
    for a, b in zip(cu[:-1], cu[1:]):
        if b == a:
            continue
        for h in range(H):
            dx[0, h, a:b] = bwd_unit(xt[0, h, a:b], xs[0, h, a:b],
                                     None if g is None else g[0, h, a:b], causal, scale, slab)
    return dx
