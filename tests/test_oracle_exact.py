"""Pins of the oracle's exact-rounding helpers (binary32 rounding of rationals
and the exactly rounded mean used by double quantization)."""

from fractions import Fraction

import numpy as np
import pytest

from oracle import exact


def test_rn32_matches_numpy_cast_of_doubles():
    """numpy's float64 -> float32 cast is correctly rounded (ties to even):
    an independent implementation for every rational that is a double."""
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(3000),
        rng.standard_normal(500) * 1e-39,          # binary32 subnormal range
        rng.standard_normal(500) * 1e30,
        np.ldexp(rng.integers(1, 2 ** 30, 500).astype(np.float64), -29),
    ])
    for v in vals:
        assert exact.rn32(Fraction(float(v))) == np.float32(v), v


def test_rn32_ties_to_even():
    one = Fraction(1)
    assert exact.rn32(one + Fraction(1, 2 ** 24)) == np.float32(1.0)
    assert exact.rn32(one + Fraction(3, 2 ** 24)) == np.float32(1.0 + 2.0 ** -22)
    assert exact.rn32(-(one + Fraction(3, 2 ** 24))) == np.float32(-(1.0 + 2.0 ** -22))
    assert exact.rn32(Fraction(1, 2 ** 150)) == np.float32(0.0)               # tie below min subnormal
    assert exact.rn32(Fraction(3, 2 ** 150)) == np.float32(2.0 ** -148)


def test_rn32_is_nearest_by_brute_force():
    """For arbitrary rationals: no binary32 neighbour is strictly closer, and a
    tie picks the even significand."""
    rng = np.random.default_rng(2)
    for _ in range(2000):
        x = Fraction(int(rng.integers(-10 ** 12, 10 ** 12)), int(rng.integers(1, 10 ** 9)))
        r = exact.rn32(x)
        if x == 0:
            assert r == 0
            continue
        for nb in (np.nextafter(r, np.float32(np.inf)), np.nextafter(r, np.float32(-np.inf))):
            dr, dn = abs(Fraction(float(r)) - x), abs(Fraction(float(nb)) - x)
            assert dr < dn or (dr == dn and (int(np.float32(r).view(np.uint32)) & 1) == 0)


def test_exact_mean_closed_forms():
    assert exact.exact_mean_f32(np.full(1000, 0.1, np.float32)) == np.float32(0.1)
    assert exact.exact_mean_f32(np.array([1.0, 2.0], np.float32)) == np.float32(1.5)
    # 2^24 + 1 + 1: a naive binary32 running sum loses both ones
    v = np.array([2.0 ** 24, 1.0, 1.0], np.float32)
    assert exact.exact_mean_f32(v) == np.float32((2.0 ** 24 + 2.0) / 3.0)
    # integers k/8: the double sum is exact, so numpy gives the exact mean too
    rng = np.random.default_rng(3)
    ints = rng.integers(0, 2 ** 20, 5001)
    v = (ints / 8.0).astype(np.float32)
    assert exact.exact_mean_f32(v) == exact.rn32(Fraction(int(ints.sum()), 8 * v.size))
    assert exact.exact_mean_f32(v) == np.float32(np.sum(v.astype(np.float64)) / v.size)


def test_exact_mean_is_order_independent():
    rng = np.random.default_rng(4)
    v = (np.abs(rng.standard_normal(4097)) * np.exp(rng.uniform(-20, 20, 4097))).astype(np.float32)
    assert exact.exact_mean_f32(v) == exact.exact_mean_f32(v[::-1].copy())
    assert exact.exact_mean_f32(v) == exact.exact_mean_f32(rng.permutation(v))


def test_exact_mean_rejects_empty():
    with pytest.raises(ValueError):
        exact.exact_mean_f32(np.zeros(0, np.float32))
