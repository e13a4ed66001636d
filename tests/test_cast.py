"""The optional bfloat16 copy of dX_s (relkl_cast_bf16).

CPU: the oracle's round-to-nearest-even (oracle.cast) is pinned to hand-worked
ties, to PyTorch's own float32 -> bfloat16 conversion, and to the rounding
invariant (the result is the nearer of the two neighbouring bf16 values, the
even one on a tie); the entry point's argument checks need no GPU.
GPU: the kernel's output equals the oracle bit for bit on every finite value,
keeps NaN a NaN, and covers the vector body, the ragged tail and unaligned
arrays (which take the element-wise kernel).
"""
import ctypes

import numpy as np
import pytest
import torch

from attention_relation_kl_b200 import _abi
from oracle import cast


def _values(n, seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(n) * np.exp2(rng.integers(-140, 128, n))).astype(np.float32)
    x[::97] = np.float32(1.0) + np.float32(2.0 ** -8) * rng.integers(0, 512, x[::97].size)  # ties
    x[1::101] = np.uint32(0x7F7F8000).view(np.float32)   # halfway above the largest bf16: infinity
    x[2::103] = np.float32(1e-40)                  # subnormal
    x[3::107] = -0.0
    return x


# ----------------------------------------------------------------- oracle pins
def test_hand_worked_ties_and_edges():
    bits = np.array([0x7F7F0000, 0x7F7F7FFF, 0x7F7F8000, 0x00008000, 0x00018000], np.uint32)
    x = np.concatenate([np.array([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20,
                                  -(1 + 2 ** -8), 3.4028235e38, 2 ** -126, 0.0, -0.0], np.float32),
                        bits.view(np.float32)])
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: the even one (1); 1 + 3 2^-8 halfway
    # between 1 + 2^-7 and 1 + 2^-6: the even one (0x3F82); the largest finite bf16
    # (0x7F7F) stays, just below halfway above it rounds down, halfway rounds to infinity;
    # subnormal ties go to the even neighbour (0 and 0x0002)
    want = [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xBF80, 0x7F80, 0x0080, 0x0000, 0x8000,
            0x7F7F, 0x7F7F, 0x7F80, 0x0000, 0x0002]
    assert [int(v) for v in cast.to_bf16_bits(x)] == want
    assert np.isnan(cast.bf16_bits_to_float(cast.to_bf16_bits(np.array([np.nan], np.float32))))


def test_matches_torch_conversion():
    x = _values(200_000, 3)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(cast.to_bf16_bits(x), ref)


def test_nearest_neighbour_invariant():
    x = _values(50_000, 4)
    x = x[np.isfinite(x) & (np.abs(x) < 3.38e38)]
    y = cast.bf16_bits_to_float(cast.to_bf16_bits(x)).astype(np.float64)
    lo = cast.bf16_bits_to_float((x.view(np.uint32) >> 16).astype(np.uint16)).astype(np.float64)
    hi = cast.bf16_bits_to_float(((x.view(np.uint32) >> 16) + 1).astype(np.uint16)).astype(np.float64)
    xd = x.astype(np.float64)
    assert np.all((y == lo) | (y == hi))
    err, other = np.abs(y - xd), np.abs(np.where(y == lo, hi, lo) - xd)
    assert np.all(err <= other)
    tie = err == other
    assert np.all((cast.to_bf16_bits(x[tie]) & 1) == 0)


# ----------------------------------------------------------- argument checks
def test_cast_validation_without_a_gpu():
    lib = _abi.lib()
    inv = _abi.RELKL_ERR_INVALID
    buf = (ctypes.c_float * 16)()
    out = (ctypes.c_uint16 * 16)()
    assert lib.relkl_cast_bf16(None, None, 0, None) == 0
    assert lib.relkl_cast_bf16(buf, out, -1, None) == inv
    assert lib.relkl_cast_bf16(None, out, 4, None) == inv
    assert lib.relkl_cast_bf16(buf, None, 4, None) == inv
    assert lib.relkl_cast_bf16(buf, ctypes.byref(buf, 2), 4, None) == inv      # overlapping
    assert lib.relkl_cast_bf16(ctypes.byref(buf, 1), out, 4, None) == inv      # misaligned src


# --------------------------------------------------------------- GPU parity
@pytest.mark.gpu
@pytest.mark.parametrize("n,src_off,dst_off", [(0, 0, 0), (1, 0, 0), (7, 0, 0), (8, 0, 0),
                                               (9, 0, 0), (1_000_003, 0, 0), (100_000, 1, 0),
                                               (100_000, 0, 1), (4_194_304, 0, 0)])
def test_cast_matches_oracle(n, src_off, dst_off):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import attention_relation_kl_b200 as rk
    x = _values(n, n + 7)
    x[5::211] = np.nan
    x[6::223] = np.inf
    src = torch.empty(n + src_off, dtype=torch.float32, device="cuda")
    src[src_off:] = torch.from_numpy(x).cuda()
    dst = torch.full((n + dst_off,), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    rk.relkl_cast_bf16(src[src_off:], out=dst[dst_off:])
    torch.cuda.synchronize()
    got = dst.view(torch.int16).cpu().numpy().astype(np.uint16)
    assert np.all(got[:dst_off] == 0xFFFF)          # nothing written before the output
    got = got[dst_off:]
    want = cast.to_bf16_bits(x)
    nan = np.isnan(x)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.all(np.isnan(cast.bf16_bits_to_float(got[nan])))


@pytest.mark.gpu
def test_backward_bf16_output_is_the_rounded_float32_gradient():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import attention_relation_kl_b200 as rk
    import workload
    w = workload.tiny_custom(N=700, d=128, dtype="bf16", seed=11, B=1, H=2)
    xt, xs = (t.cuda() for t in workload.generate(w)["q"])
    _, st = rk.relkl_fwd(xt, xs)
    # the float32 result of the same call (reduce-adds make the last bits of two
    # calls' results differ)
    dx32 = torch.empty(xs.shape, dtype=torch.float32, device=xs.device)
    dx16 = rk.relkl_bwd(xt, xs, st, dx_s=dx32, dx_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert dx16.dtype == torch.bfloat16 and dx16.shape == dx32.shape
    want = cast.to_bf16_bits(dx32.cpu().numpy().ravel())
    got = dx16.view(torch.int16).cpu().numpy().astype(np.uint16).ravel()
    assert np.array_equal(got, want)
