"""Pins of the oracle's NF-k codebook against what the pages and mathematics fix.

"QLoRA: Efficient Finetuning of Quantized LLMs", section "Method", paragraph
"4-bit NormalFloat Quantization".
"""

import numpy as np
import pytest
from scipy import special

from oracle import codebook
from tests.conftest import read_golden

FIG = {k: float(v) for k, v in read_golden("paper_figures.txt")}


@pytest.mark.parametrize("p,x", [(float(a), float(b)) for a, b in read_golden("normal_quantiles.txt")])
def test_norm_ppf_textbook_values(p, x):
    assert codebook.norm_ppf(p) == pytest.approx(x, abs=2e-15, rel=2e-15)


def test_norm_ppf_against_library_routine():
    for p in np.linspace(0.001, 0.999, 137):
        assert codebook.norm_ppf(float(p)) == pytest.approx(float(special.ndtri(p)), rel=1e-13, abs=1e-13)


def test_nf4_structure_matches_the_page():
    q = codebook.nf4_codebook()
    assert q.dtype == np.float32
    assert q.size == FIG["codebook_size"] == 2 ** FIG["k_bits"]
    assert np.all(np.diff(q) > 0), "strictly increasing"
    assert q[0] == FIG["range_lo"] and q[-1] == FIG["range_hi"], "normalized into [-1, 1]"
    assert np.count_nonzero(q == 0.0) == 1, "exactly one exact zero"
    # 2^(k-1) negative-part quantiles and 2^(k-1)+1 positive-part quantiles, the
    # shared zero counted once: 7 negative, 1 zero, 8 positive
    assert np.count_nonzero(q < 0) == FIG["negative_part_quantiles"] - 1
    assert np.count_nonzero(q > 0) == FIG["positive_part_quantiles"] - 1
    assert int(np.flatnonzero(q == 0.0)[0]) == 7


def test_nf4_values_are_equally_spaced_quantiles():
    """Undo the normalization with an independent Phi (scipy): the positive
    values must sit at 8 equal probability steps from 1/2 to 1 - delta, the
    negative ones at 7 equal steps (step (1) of the construction)."""
    delta = codebook.DEFAULT_DELTA
    q = codebook.nfk_codebook_f64(4, delta)
    top = special.ndtri(1.0 - delta)
    p = special.ndtr(q * top)
    pos, neg = p[q > 0], p[q < 0]
    np.testing.assert_allclose(np.diff(np.concatenate([[0.5], pos])), (0.5 - delta) / 8, rtol=1e-9)
    np.testing.assert_allclose(np.diff(np.concatenate([neg, [0.5]])), (0.5 - delta) / 7, rtol=1e-9)
    assert p[-1] == pytest.approx(1.0 - delta, rel=1e-12)
    assert p[0] == pytest.approx(delta, rel=1e-9)


def test_nf4_binary32_values_are_the_rounded_float64_construction():
    q64 = codebook.nfk_codebook_f64(4)
    assert np.array_equal(codebook.nf4_codebook(), q64.astype(np.float32))


@pytest.mark.parametrize("k", [2, 3, 5])
def test_nfk_general_k(k):
    q = codebook.nfk_codebook_f64(k)
    assert q.size == 2 ** k
    assert q[0] == -1.0 and q[-1] == 1.0
    assert np.count_nonzero(q == 0.0) == 1
    assert np.count_nonzero(q < 0) == 2 ** (k - 1) - 1
    assert np.all(np.diff(q) > 0)


def test_int4_table_structure():
    """Int4 as an absmax code: sixteen strictly increasing values, the zero at
    index 8 (two's-complement order), +-1 exactly at the levels +-7, one
    level below -1, and every value within a binary32 rounding of an integer
    multiple of 1/7 (checked in exact rationals)."""
    from fractions import Fraction
    q = codebook.int4_codebook()
    assert q.dtype == np.float32 and q.size == 16
    assert np.all(np.diff(q) > 0)
    assert np.count_nonzero(q == 0.0) == 1 and q[8] == 0.0
    assert q[1] == -1.0 and q[15] == 1.0 and q[0] < -1.0
    for j, v in enumerate(q):
        level = Fraction(j - 8, 7)
        ulp = Fraction(float(np.spacing(np.float32(abs(v)) if v else np.float32(1e-38))))
        assert abs(Fraction(float(v)) - level) <= ulp / 2, (j, float(v))


def test_e2m1_values_match_the_ocp_table():
    rows = read_golden("e2m1_spec.txt")
    assert len(rows) == 16
    for code, val in rows:
        got = codebook.e2m1_value(int(code, 16))
        assert got == float(val) and np.signbit(got) == val.startswith("-"), code


def test_fp4_table_structure():
    q = codebook.fp4_codebook()
    assert q.dtype == np.float32 and len(q) == 16
    assert np.all(np.diff(q.astype(np.float64)) > 0), "strictly increasing"
    assert np.count_nonzero(q == 0) == 1 and q[8] == 0
    assert q[1] == -1.0 and q[15] == 1.0 and q[0] < -1.0
    # the distinct E2M1 values over 6, each one binary32 rounding of the exact quotient
    for v, want in zip(q[1:], [-6, -4, -3, -2, -1.5, -1, -0.5, 0, 0.5, 1, 1.5, 2, 3, 4, 6]):
        assert v == np.float32(want / 6.0)
    # the pad below -1 is never the nearest value of anything in [-1, 1]
    assert (q[0] + q[1]) / 2 < -1.0



@pytest.mark.parametrize("k", [2, 3, 4])
def test_nfk_tables(k):
    """NF-k in the 16-entry table: 2^k NormalFloat values with the page's
    structure (2^(k-1) negative, one zero, 2^(k-1) positive, +-1 at the ends),
    equally spaced probabilities behind them (undone with scipy's Phi), and
    never-nearest pads beyond +-1."""
    t = codebook.nfk_table(k)
    assert len(t) == 16 and np.all(np.diff(t.astype(np.float64)) > 0)
    n = 2 ** k
    pad = (16 - n) // 2
    v = t[pad:pad + n].astype(np.float64)
    assert v[0] == -1.0 and v[-1] == 1.0 and np.count_nonzero(v == 0) == 1
    assert np.count_nonzero(v < 0) == n // 2 - 1 and np.count_nonzero(v > 0) == n // 2
    if pad:
        assert (t[pad - 1] + t[pad]) / 2 < -1.0 and (t[pad + n - 1] + t[pad + n]) / 2 > 1.0
    d = codebook.nfk_default_delta(k)
    top = special.ndtri(1.0 - d)
    for side in (v[v > 0], -v[v < 0]):
        # the zero (probability 1/2) and the side's values, undone with Phi
        steps = np.diff(np.sort(np.concatenate([[0.5], special.ndtr(side * top)])))
        np.testing.assert_allclose(steps, steps[0], rtol=1e-6)
    if k == 4:
        assert np.array_equal(t.view(np.uint32), codebook.nf4_codebook().view(np.uint32))
