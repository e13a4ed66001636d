"""bfloat16 rounding of float32 values, written out from the format's definition.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

bfloat16 keeps the sign, the 8 exponent bits and the top 7 mantissa bits of a
float32.  Round to nearest, ties to even: add 0x7FFF plus the lowest kept bit
to the 32-bit pattern and drop the low 16 bits.  The carry moves into the
exponent when the mantissa overflows, and from the largest finite values it
reaches the infinity pattern, as IEEE rounding requires.  A NaN stays a NaN
(quiet, sign kept).  This restates the optional bf16 copy of dX_s that
follows the float32 accumulation of the path's backward (the pages fix the
gradient's float32 accumulation only; the copy is a storage convenience).
"""
import numpy as np


def to_bf16_bits(x) -> np.ndarray:
    """uint16 bit patterns of x (float32 array) rounded to bfloat16, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    r[nan] = ((u[nan] >> 16).astype(np.uint16) | 0x0040)   # quiet NaN, sign kept
    return r


def bf16_bits_to_float(b) -> np.ndarray:
    """float32 values of uint16 bfloat16 patterns."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
