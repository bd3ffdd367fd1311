"""The CUDA library's exactly-rounded mean (header shared by the quantize
kernels), compiled for the host and checked against the oracle's rational
arithmetic.  Reading of "Double Quantization" (QLoRA paper, section "Method"):
the subtracted mean is the binary32 nearest to the exact mean of all c1."""

import ctypes
import os
import subprocess

import numpy as np
import pytest

from oracle import exact

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("em") / "libem.so")
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared",
                           os.path.join(HERE, "helpers", "exact_mean_host.cpp"), "-o", out])
    l = ctypes.CDLL(out)
    l.host_exact_mean_bits.restype = ctypes.c_uint32
    l.host_exact_mean_bits.argtypes = [ctypes.c_void_p, ctypes.c_int64]
    return l


def _mean(lib, v):
    v = np.ascontiguousarray(v, np.float32)
    return np.uint32(lib.host_exact_mean_bits(v.ctypes.data, v.size)).view(np.float32)


@pytest.mark.parametrize("case", range(12))
def test_matches_oracle_on_random_sets(lib, case):
    rng = np.random.default_rng(100 + case)
    n = int(rng.integers(1, 20000))
    kind = case % 4
    if kind == 0:      # absmax-like constants of N(0, 0.02) blocks
        v = np.abs(rng.standard_normal((n, 64)) * 0.02).max(axis=1)
    elif kind == 1:    # wide dynamic range
        v = np.abs(rng.standard_normal(n)) * np.exp(rng.uniform(-80, 80, n))
    elif kind == 2:    # subnormals and zeros mixed in
        v = np.abs(rng.standard_normal(n)) * 1e-39
        v[rng.random(n) < 0.3] = 0
    else:              # few distinct values, exact-tie friendly
        v = rng.integers(0, 5, n) * 0.25
    v = v.astype(np.float32)
    assert _mean(lib, v) == exact.exact_mean_f32(v)


def test_closed_forms(lib):
    assert _mean(lib, np.zeros(7)) == 0.0
    assert _mean(lib, np.full(3, 0.1)) == np.float32(0.1)
    assert _mean(lib, np.array([1.0, 2.0])) == np.float32(1.5)
    # ties: mean = 1 + 2^-24 (halfway) -> 1; 1 + 3*2^-24 -> 1 + 2^-22
    one = np.float32(1.0)
    up = np.nextafter(one, np.float32(2))            # 1 + 2^-23
    assert _mean(lib, np.array([one, up])) == one
    assert _mean(lib, np.array([up, np.nextafter(up, np.float32(2))])) == np.float32(1 + 2 ** -22)
    # smallest subnormal halves: mean of {2^-149, 0} is a tie between 0 and 2^-149
    tiny = np.float32(2.0 ** -149)
    assert _mean(lib, np.array([tiny, 0.0], np.float32)) == 0.0
    assert _mean(lib, np.array([tiny, tiny, 0.0], np.float32)) == tiny
    assert _mean(lib, np.array([3.0e38, 3.0e38], np.float32)) == np.float32(3.0e38)
