"""Exactly rounded helpers in Python integers (oracle side).

TEST INFRASTRUCTURE (see the package docstring).

Double quantization subtracts the mean of the first-level constants before
quantizing them ("QLoRA: Efficient Finetuning of Quantized LLMs", section
"Method", paragraph "Double Quantization"; the page stops before giving the
arithmetic).  Reading used: the mean is the binary32 number nearest to the
exact arithmetic mean of all c1 of the tensor, ties to even.  That makes it
independent of summation order, so the GPU may reduce in any order.
"""

from fractions import Fraction

import numpy as np


def _floor_log2(a: int, b: int) -> int:
    """floor(log2(a / b)) for positive integers a, b."""
    e = a.bit_length() - b.bit_length()
    if (a << -e if e < 0 else a) < (b << e if e > 0 else b):
        e -= 1
    return e


def rn32(x) -> np.float32:
    """Round a rational number (int, Fraction or exactly-converted float) to
    the nearest binary32 value, ties to even; subnormals included.  Results
    beyond the binary32 range are an error (never needed here)."""
    x = Fraction(x)
    if x == 0:
        return np.float32(0.0)
    sign = -1 if x < 0 else 1
    a, b = abs(x.numerator), x.denominator
    e = _floor_log2(a, b)                 # 2^e <= |x| < 2^(e+1)
    qexp = max(e, -126) - 23              # value of one unit in the last place
    num, den = (a << -qexp, b) if qexp < 0 else (a, b << qexp)
    q, r = divmod(num, den)
    if 2 * r > den or (2 * r == den and q & 1):
        q += 1
    if q * 2.0 ** qexp >= 2.0 ** 128:
        raise OverflowError("beyond binary32 range")
    return np.float32(sign * q * 2.0 ** qexp)   # q <= 2^24: exact conversions


def exact_mean_f32(values: np.ndarray) -> np.float32:
    """Binary32 nearest to the exact arithmetic mean of binary32 values."""
    v = np.asarray(values, dtype=np.float32).ravel()
    if v.size == 0:
        raise ValueError("mean of an empty set")
    # every binary32 is an integer multiple of 2^-149: scale exactly, sum as ints
    scaled = v.astype(np.float64) * 2.0 ** 149
    total = sum(int(s) for s in scaled.tolist())
    return rn32(Fraction(total, v.size * 2 ** 149))
