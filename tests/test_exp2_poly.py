"""The FMA-pipe 2^x of the CUDA kernels (relkl_device.cuh, exp2_poly2),
emulated bit for bit in NumPy float32: the rint-by-1.5*2^23 reduction, the
polynomial with the coefficients the header holds, and the exponent-field
insert.  Checks the relative error over the whole argument range used
(x in [-125, 0]) against the bound the header quotes."""
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "attention_relation_kl_b200", "csrc", "relkl_device.cuh")


def _coeffs(deg):
    src = open(HDR).read()
    body = src[src.index("__device__ __forceinline__ float2 exp2_poly2"):]
    body = body[:body.index("return make_float2")]
    branch = body[body.index("if constexpr (DEG == 5)"):]
    five, rest = branch.split("} else {")
    three = rest[:rest.index("\n  }\n")]
    part = five if deg == 5 else three
    vals = [float(v) for v in re.findall(r"make_float2\(([-0-9.e+]+)f,", part)]
    # Horner order in the source: highest coefficient first, ending with c1
    return np.array(vals[::-1][: deg], dtype=np.float32)  # c1..c_deg


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def emulate(x, deg):
    c = _coeffs(deg)
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = _fma32(n, np.float32(-1.0), x)
    p = np.full_like(f, c[-1])
    for k in range(deg - 2, -1, -1):
        p = _fma32(p, f, np.full_like(f, c[k]))
    p = _fma32(p, f, np.ones_like(f))
    bits = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32)


@pytest.mark.parametrize("deg,bound", [(5, 2.0e-7), (3, 1.1e-4)])
def test_exp2_poly_relative_error(deg, bound):
    rng = np.random.default_rng(deg)
    x = np.concatenate([rng.uniform(-125.0, 0.0, 200000), rng.uniform(-1.0, 0.0, 100000),
                        np.arange(-125, 1, dtype=np.float64), [-0.5, -1.5, -124.5]]).astype(np.float32)
    got = emulate(x, deg).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() <= bound, (rel.max(), x[np.argmax(rel)])
    # arguments below the clamp give tiny positive values, never garbage
    low = emulate(np.array([-126.0, -300.0, -1e30], dtype=np.float32), deg)
    assert np.all(low >= 0) and np.all(low <= 2.0 ** -124)
