"""Float64 CPU oracle for the chain rule from dX_s to the student's Q/K/V weights.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference arm may import this module.  It shares no code
with the CUDA path and is never called by the product.

What it computes.  In LinearARD only the student's Q/K/V projections are
trained (pith.science verdict page, ``minor_comments``); the relation loss
reaches them through the student's inputs X_s = RoPE_s(H_s W_x) (x in q, k;
V takes no rotation).  The pages stop at the gradient of the relation
logits; the rest is the plain chain rule:

* RoPE backward.  Rotate-half RoPE (RoFormer's rotary embedding in LLaMA's
  pairing: dimension i with i + d/2, angle pos * base^(-2i/d)) maps a pair
  (a, b) to (a cos - b sin, b cos + a sin).  Its Jacobian is that rotation, so
  the gradient of the pre-rotation vector is the transposed rotation of the
  post-rotation gradient: (g_a cos + g_b sin, g_b cos - g_a sin).
* Weight gradient.  With the heads laid side by side per token,
  X_pre[b, n, :] = H_s[b, n, :] W_x, so dW_x = sum over b, n of
  H_s[b, n, :]^T dX_pre[b, n, :] = H_s^T dX_pre over the B*N token rows.

Everything is float64 NumPy on exactly converted inputs.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

from . import dense


def as_f64(x) -> np.ndarray:
    return dense.as_f64(x)


def rope_angles(positions, d: int, base: float) -> np.ndarray:
    """Angle of pair i at each position: pos * base^(-2i/d), shape [N, d/2]."""
    if d % 2:
        raise ValueError("RoPE needs an even head dimension")
    pos = np.asarray(positions, dtype=np.float64)
    inv_freq = base ** (-np.arange(d // 2, dtype=np.float64) * 2.0 / d)
    return pos[:, None] * inv_freq[None, :]


def rope_backward(dy, positions, base: float) -> np.ndarray:
    """Gradient of the pre-rotation vectors from that of the rotated ones.

    dy: [..., N, d] gradient with respect to RoPE(x); returns [..., N, d].
    """
    g = as_f64(dy)
    d = g.shape[-1]
    ang = rope_angles(positions, d, base)
    c, s = np.cos(ang), np.sin(ang)
    ga, gb = g[..., : d // 2], g[..., d // 2:]
    return np.concatenate((ga * c + gb * s, gb * c - ga * s), axis=-1)


def heads_to_tokens(x) -> np.ndarray:
    """[B, heads, N, d] -> [B, N, heads * d]: the per-token layout of a projection."""
    a = as_f64(x)
    B, Hh, N, d = a.shape
    return a.transpose(0, 2, 1, 3).reshape(B, N, Hh * d)


def weight_grad(h, dx_tokens) -> np.ndarray:
    """dW = sum over batch and tokens of h[b, n]^T dx[b, n]: [D, cols]."""
    hh, dd = as_f64(h), as_f64(dx_tokens)
    B, N, D = hh.shape
    return hh.reshape(B * N, D).T @ dd.reshape(B * N, -1)


def projection_grads(x: Dict[str, tuple], h_s, pos_s, rope_base: float,
                     dkl: Optional[Dict[str, np.ndarray]] = None,
                     causal: bool = True) -> Dict[str, np.ndarray]:
    """dW_q, dW_k, dW_v of the student from the relation-KL gradients.

    x: {rel: (x_teacher, x_student)} [B, heads, N, d] post-RoPE; h_s: [B, N, D];
    dkl: optional upstream per-row gradients {rel: [B, heads, N]} (default 1/N).
    """
    out = {}
    for rel, (xt, xs) in x.items():
        dx = dense.bwd(xt, xs, None if dkl is None else dkl.get(rel), causal)
        if rel != "v":
            dx = rope_backward(dx, pos_s, rope_base)
        out[rel] = weight_grad(h_s, heads_to_tokens(dx))
    return out
