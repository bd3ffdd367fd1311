"""Pins of the oracle's QLoRA linear: brute-force loops, finite differences of
the forward, and the special cases that reduce to a plain product.

mbrenndoerfer.com QLoRA essay, section "Low-Rank Adaptation (LoRA)"
(x_out = (W_q + BA) x_in); "QLoRA: Efficient Finetuning of Quantized LLMs",
section "Method" (16-bit matmul with the dequantized weight) and abstract
(gradients flow through the frozen 4-bit weight into the adapters only).
"""

import numpy as np

from oracle import linear


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_forward_against_triple_loops():
    rng = np.random.default_rng(12)
    M, K, N, r, s = 3, 8, 5, 2, 0.75
    X, W, A, B = _rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K), _rand(rng, N, r)
    Y = linear.forward(X, W, A, B, s)
    for m in range(M):
        for n in range(N):
            ref = 0.0
            for k in range(K):
                dw = sum(B[n, j] * A[j, k] for j in range(r))          # (B A)[n, k]
                ref += (W[n, k] + s * dw) * X[m, k]
            assert abs(Y[m, n] - ref) < 1e-12


def test_backward_against_finite_differences():
    rng = np.random.default_rng(13)
    M, K, N, r, s = 4, 6, 5, 3, 0.5
    X, W, A, B, dY = (_rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K),
                      _rand(rng, N, r), _rand(rng, M, N))
    dX, dA, dB = linear.backward(X, W, A, B, s, dY)

    def loss(X_, A_, B_):
        return float(np.sum(dY * linear.forward(X_, W, A_, B_, s)))

    h = 1e-6
    for name, P, G in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        for idx in np.ndindex(P.shape):
            Pp, Pm = P.copy(), P.copy()
            Pp[idx] += h
            Pm[idx] -= h
            args_p = {"X": (Pp, A, B), "A": (X, Pp, B), "B": (X, A, Pp)}[name]
            args_m = {"X": (Pm, A, B), "A": (X, Pm, B), "B": (X, A, Pm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - G[idx]) < 1e-6 * max(1.0, abs(fd)), (name, idx)


def test_zero_adapter_and_zero_scale_reduce_to_plain_product():
    rng = np.random.default_rng(14)
    M, K, N, r = 5, 16, 7, 4
    X, W, A, dY = _rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K), _rand(rng, M, N)
    B0 = np.zeros((N, r))
    np.testing.assert_allclose(linear.forward(X, W, A, B0, 2.0), X @ W.T, rtol=0, atol=1e-12)
    dX, dA, dB = linear.backward(X, W, A, B0, 2.0, dY)
    np.testing.assert_allclose(dX, dY @ W, atol=1e-12)
    assert np.all(dA == 0)
    B = _rand(rng, N, r)
    np.testing.assert_allclose(linear.forward(X, W, A, B, 0.0), X @ W.T, atol=1e-12)
    dX, dA, dB = linear.backward(X, W, A, B, 0.0, dY)
    assert np.all(dA == 0) and np.all(dB == 0)


def test_row_helpers_match_full_products():
    rng = np.random.default_rng(15)
    M, K, N, r, s = 9, 64, 12, 4, 0.25
    X, W, A, B, dY = (_rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K),
                      _rand(rng, N, r), _rand(rng, M, N))
    rows = [0, 3, 8]
    np.testing.assert_allclose(linear.forward_rows(X, W, A, B, s, rows),
                               linear.forward(X, W, A, B, s)[rows], atol=1e-12)
    np.testing.assert_allclose(linear.backward_dx_rows(W, A, B, s, dY, rows),
                               linear.backward(X, W, A, B, s, dY)[0][rows], atol=1e-12)


def test_weight_grad_helper_matches_full_backward():
    rng = np.random.default_rng(16)
    M, K, N, r, s = 11, 64, 24, 8, 0.25
    X, W, A, B, dY = (_rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K),
                      _rand(rng, N, r), _rand(rng, M, N))
    _, dA, dB = linear.backward(X, W, A, B, s, dY)
    gA, gB = linear.backward_weight_grads(X, A, B, s, dY)
    np.testing.assert_allclose(gA, dA, rtol=0, atol=1e-12)
    np.testing.assert_allclose(gB, dB, rtol=0, atol=1e-12)
    # and against brute-force sums over tokens: dA[j,k] = s sum_m (sum_n dY[m,n] B[n,j]) X[m,k]
    for j in range(r):
        for k in (0, 17, 63):
            ref = s * sum(sum(dY[m, n] * B[n, j] for n in range(N)) * X[m, k] for m in range(M))
            assert abs(gA[j, k] - ref) < 1e-10


def test_dropout_gradients_against_finite_differences():
    """With the unrounded dropped-out input, the backward pass is the exact
    derivative of the forward pass in X, A and B."""
    rng = np.random.default_rng(17)
    M, K, N, r, s, p = 4, 8, 5, 3, 0.5, 0.25
    X, W, A, B, dY = (_rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K), _rand(rng, N, r), _rand(rng, M, N))
    mask = rng.random((M, K)) >= p
    sc = np.float64(linear.dropout_scale(p))

    def fwd(X_, A_, B_):
        return linear.forward_dropout(X_, W, A_, B_, s, X_ * mask * sc)

    def loss(X_, A_, B_):
        return float(np.sum(dY * fwd(X_, A_, B_)))

    dX, dA, dB = linear.backward_dropout(X, W, A, B, s, dY, X * mask * sc, mask, p)
    h = 1e-6
    for name, P, G in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        for idx in np.ndindex(P.shape):
            Pp, Pm = P.copy(), P.copy()
            Pp[idx] += h
            Pm[idx] -= h
            ap = {"X": (Pp, A, B), "A": (X, Pp, B), "B": (X, A, Pp)}[name]
            am = {"X": (Pm, A, B), "A": (X, Pm, B), "B": (X, A, Pm)}[name]
            fd = (loss(*ap) - loss(*am)) / (2 * h)
            assert abs(fd - G[idx]) < 1e-6 * max(1.0, abs(fd)), (name, idx)


def test_dropout_special_cases():
    rng = np.random.default_rng(18)
    M, K, N, r, s = 3, 16, 6, 2, 2.0
    X = np.clip(np.round(rng.standard_normal((M, K)) * 64) / 64, -3.9, 3.9)   # exact in bf16
    W, A, B, dY = _rand(rng, N, K), _rand(rng, r, K), _rand(rng, N, r), _rand(rng, M, N)
    # p = 0 with every input kept is the plain layer (scale 1: x_d = bf16(x) = x for bf16-exact x)
    keep = np.ones((M, K), bool)
    Xb = linear.dropout_input(X.astype(np.float32), keep, 0.0, bf16_round=False)
    np.testing.assert_array_equal(Xb, X)
    np.testing.assert_allclose(linear.forward_dropout(X, W, A, B, s, Xb), linear.forward(X, W, A, B, s), atol=1e-12)
    for a, b in zip(linear.backward_dropout(X, W, A, B, s, dY, Xb, keep, 0.0), linear.backward(X, W, A, B, s, dY)):
        np.testing.assert_allclose(a, b, atol=1e-12)
    # everything dropped: the adapter branch vanishes
    drop = np.zeros((M, K), bool)
    Xd = linear.dropout_input(X.astype(np.float32), drop, 0.5)
    np.testing.assert_allclose(linear.forward_dropout(X, W, A, B, s, Xd), X @ W.T, atol=1e-12)
    dX, dA, dB = linear.backward_dropout(X, W, A, B, s, dY, Xd, drop, 0.5)
    assert not dA.any() and not dB.any()
    np.testing.assert_allclose(dX, dY @ W, atol=1e-12)
    # the scale of p = 0.5 is exactly 2 and the bf16 rounding of x * 2 is exact
    half = rng.random((M, K)) >= 0.5
    np.testing.assert_array_equal(linear.dropout_input(X.astype(np.float32), half, 0.5), X * 2 * half)
    # the scale of p = 0.05: RN32(1 / RN32(0.95)), checked against the correctly
    # rounded float32 division of numpy
    assert linear.dropout_scale(0.05) == np.float32(1.0) / np.float32(0.95)
    assert linear.dropout_scale(0.1) == np.float32(1.0) / np.float32(0.9)


def test_error_metrics():
    ref = np.array([[3.0, 4.0]])
    assert linear.rel_frobenius(ref, ref) == 0.0
    assert linear.rel_frobenius(ref + np.array([[0.0, 0.5]]), ref) == 0.1
    assert linear.max_abs(ref + 0.25, ref) == 0.25
