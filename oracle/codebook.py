"""NF-k codebook straight from the construction on the page (oracle side).

TEST INFRASTRUCTURE (see the package docstring).

"QLoRA: Efficient Finetuning of Quantized LLMs", section "Method", paragraph
"4-bit NormalFloat Quantization":
  (1) estimate quantiles of a theoretical N(0, 1) distribution,
  (2) normalize the values into [-1, 1],
  asymmetric construction: 2^(k-1) quantiles for the negative part and
  2^(k-1) + 1 for the positive part; unify both sets and remove one of the two
  zeros that occur in both.  (The page's superscripts were lost in
  extraction; "2k - 1" there is 2^(k-1).)

The equation that fixes the probabilities is missing from the page.  Reading
used here: each side takes equally spaced probabilities from 1 - delta down to
1/2, where delta is the tail probability of the outermost value; the default
delta = (1/(2*16) + 1/(2*15)) / 2 puts the outermost value at the centre of
the outermost equal-mass bin, averaged over the 16- and 15-level halves.

Phi^-1 is computed here by bisection on Phi(x) = erfc(-x / sqrt 2) / 2 with
libm's erfc: a method deliberately different from the one in the CUDA
library's host code.
"""

import math

import numpy as np

DEFAULT_DELTA = 0.5 * (1.0 / 32.0 + 1.0 / 30.0)


def norm_cdf(x: float) -> float:
    """Phi(x) of N(0, 1)."""
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def norm_ppf(p: float) -> float:
    """Phi^-1(p) by bisection to adjacent doubles; Phi^-1(1/2) = 0 exactly
    (symmetry of N(0, 1))."""
    if not 0.0 < p < 1.0:
        raise ValueError("p must lie in (0, 1)")
    if p == 0.5:
        return 0.0
    lo, hi = -40.0, 40.0
    for _ in range(4000):
        mid = 0.5 * (lo + hi)
        if mid == lo or mid == hi:
            break
        if norm_cdf(mid) < p:
            lo = mid
        else:
            hi = mid
    # the crossing lies in [lo, hi], two adjacent doubles: take the closer one
    return lo if abs(norm_cdf(lo) - p) <= abs(norm_cdf(hi) - p) else hi


def _probabilities(a: float, b: float, n: int):
    """n equally spaced probabilities from a to b, both ends included."""
    return [a + (b - a) * i / (n - 1) if i < n - 1 else b for i in range(n)]


def nfk_codebook_f64(k: int = 4, delta: float = DEFAULT_DELTA) -> np.ndarray:
    """The 2^k NF-k values in float64, ascending, in [-1, 1]."""
    top = norm_ppf(1.0 - delta)
    pos = [norm_ppf(p) for p in _probabilities(1.0 - delta, 0.5, 2 ** (k - 1) + 1)]
    neg = [-norm_ppf(p) for p in _probabilities(1.0 - delta, 0.5, 2 ** (k - 1))]
    # both sets end in 0: unify and drop one of the two zeros
    values = pos + neg[:-1]
    assert neg[-1] == 0.0 and pos[-1] == 0.0
    values = sorted(v / top for v in values)
    return np.array(values, dtype=np.float64)


def nfk_default_delta(k: int) -> float:
    """The default tail probability of the NF-k reading above for any k: the
    centre of the outermost equal-mass bin, averaged over the 2^k- and
    (2^k - 1)-level halves (for k = 4 this is DEFAULT_DELTA)."""
    n = 2 ** k
    return 0.5 * (1.0 / (2 * n) + 1.0 / (2 * (n - 1)))


def nfk_table(k: int, delta: float = None) -> np.ndarray:
    """NF-k (k = 2, 3, 4) as the 16 binary32 values the 4-bit codec stores:
    the 2^k NF-k values (rounded once), with 16 - 2^k padding values beyond
    +-1 (half below -1 at -1 - i/4, half above +1 at 1 + i/4, i = 1, 2, ...),
    which are never the nearest value of anything in [-1, 1]; for k = 4 the
    table is NF4 itself."""
    if k not in (2, 3, 4):
        raise ValueError("k must be 2, 3 or 4")
    d = nfk_default_delta(k) if delta is None else delta
    vals = list(nfk_codebook_f64(k, d).astype(np.float32))
    half = (16 - 2 ** k) // 2
    below = [np.float32(-1.0 - i / 4.0) for i in range(half, 0, -1)]
    above = [np.float32(1.0 + i / 4.0) for i in range(1, half + 1)]
    return np.array(below + vals + above, dtype=np.float32)


def nf4_codebook(delta: float = DEFAULT_DELTA) -> np.ndarray:
    """NF4 as the 16 binary32 values the codec stores (rounded once)."""
    return nfk_codebook_f64(4, delta).astype(np.float32)


def int4_codebook() -> np.ndarray:
    """4-bit integers as an absmax code.  The paper's introduction, item (1),
    names 4-bit integers as the data type NF4 is compared with but does not
    define them.  Reading: the sixteen two's-complement values -8 .. 7 over
    the level count 7, so that +-7 carry the block's absmax (one binary32
    rounding of each exact quotient).  -8/7 lies below -1 and never wins."""
    return np.array([np.float32(float(j) / 7.0) for j in range(-8, 8)], dtype=np.float32)


def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code: sign bit 3, exponent bits 2..1 (bias 1),
    mantissa bit 0; exponent field 0 is the subnormal range (m * 2^-1)."""
    sign = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    mag = m * 0.5 if e == 0 else (1.0 + 0.5 * m) * 2.0 ** (e - 1)
    return sign * mag


def fp4_codebook() -> np.ndarray:
    """4-bit floats as an absmax code.  The paper's introduction, item (1),
    names 4-bit floats as the other data type NF4 is compared with but does not
    define them.  Reading: the E2M1 values (the 4-bit float of the OCP
    microscaling formats) over their largest magnitude 6, so that +-6 carry the
    block's absmax.  E2M1 holds 15 distinct values (+0 and -0 coincide); the
    sixteenth entry is -8/6, the magnitude one exponent step beyond 6, which
    lies below -1 and never wins, as -8/7 in the Int4 table."""
    vals = sorted({e2m1_value(c) for c in range(16)})      # -0 and +0 collapse
    assert len(vals) == 15
    top = max(abs(v) for v in vals)
    return np.array([np.float32(-8.0 / top)] + [np.float32(v / top) for v in vals], dtype=np.float32)

