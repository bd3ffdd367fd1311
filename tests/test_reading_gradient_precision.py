"""The precision reading for the weight gradients, checked in float64 on the
benchmark's input distributions (weights N(0, 0.02), X and dY N(0, 1), B
N(0, 0.01), r = 64, alpha = 16, 4096 tokens).

dA = G^T X with G = s dY B.  Rounding G once to bfloat16 (8 significant bits)
before the product already moves dA by more than the 2e-2 max-abs bar at
4096 tokens, because dA's entries grow like sqrt(tokens); carrying G as a
bf16 pair (hi = bf16(G), lo = bf16(G - hi), about 16 significant bits) keeps
the same product well inside the bar.  This is why the library feeds the
weight-gradient products hi + lo halves.
"""

import numpy as np

from oracle import codec


def _bf16(x):
    return codec.bf16_bits_to_f32(codec.bf16_rne(np.asarray(x, np.float32))).astype(np.float64)


def test_single_bf16_g_misses_the_bar_and_a_hi_lo_pair_meets_it():
    rng = np.random.default_rng(5)
    M, N, K, r, s = 4096, 4096, 256, 64, 16.0 / 64
    dY = rng.standard_normal((M, N), dtype=np.float32).astype(np.float64)
    B = (rng.standard_normal((N, r), dtype=np.float32) * 0.01).astype(np.float64)
    X = _bf16(rng.standard_normal((M, K), dtype=np.float32))
    G = s * (dY @ B)                      # exact enough in float64 for this purpose
    dA = G.T @ X
    assert np.abs(dA).max() > 30          # entries grow like sqrt(M): about 10 std
    g_hi = _bf16(G)
    g_lo = _bf16(G - g_hi)
    err_single = np.abs(g_hi.T @ X - dA).max()
    err_pair = np.abs((g_hi + g_lo).T @ X - dA).max()
    assert err_single > 2e-2, err_single
    assert err_pair < 2e-2 / 50, err_pair
