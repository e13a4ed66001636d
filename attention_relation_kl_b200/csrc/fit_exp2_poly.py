"""Fit the polynomials the CUDA kernels use for 2^f on [-1/2, 1/2].

    python attention_relation_kl_b200/csrc/fit_exp2_poly.py

2^x = 2^n * 2^f with n = rint(x), f = x - n in [-1/2, 1/2] (Cody and Waite's
argument reduction); 2^f is approximated by p(f) = 1 + c1 f + ... + ck f^k,
fitted for minimax *relative* error by iteratively reweighted least squares
on Chebyshev points.  Prints float32 coefficients and the relative error of a
float32 Horner evaluation, which relkl_device.cuh quotes.
"""
import numpy as np


def fit(deg: int, iters: int = 80):
    f = 0.5 * np.cos(np.linspace(0.0, np.pi, 6001))
    y = np.exp2(f)
    V = np.stack([f ** k for k in range(1, deg + 1)], 1)
    w = np.ones_like(f)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(V * (w / y)[:, None], (y - 1.0) * (w / y), rcond=None)
        err = (1.0 + V @ c - y) / y
        w = w * (1.0 + 50.0 * np.abs(err) / np.abs(err).max())
        w /= w.mean()
    return c.astype(np.float32)


def horner_f32(c, f):
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)
    return (p * f + np.float32(1.0)).astype(np.float32)


if __name__ == "__main__":
    f = np.random.default_rng(0).uniform(-0.5, 0.5, 400000).astype(np.float32)
    for deg in (3, 4, 5):
        c = fit(deg)
        rel = np.abs(horner_f32(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1).max()
        print(f"degree {deg}: rel err {rel:.3e}  c1..c{deg} = " +
              ", ".join(f"{float(v):.9e}f" for v in c))
