"""Pins of the oracle's transformer block: central finite differences of the
whole block (input and every adapter), and closed forms of its parts
(RMSNorm of a constant row, RoPE at position 0 and as a rotation, attention
over one token and over identical keys).

"QLoRA: Efficient Finetuning of Quantized LLMs", Introduction (adapters at
every layer, gradient checkpointing); the block layout is the LLaMA reading
stated in oracle/block.py."""

import numpy as np

from oracle import block

CFG = dict(batch=2, seq=5, heads=2, head_dim=4, r=2, scale=0.7, eps=1e-6, rope_base=10000.0)
HIDDEN, INTER = 8, 12


def _params(seed):
    rng = np.random.default_rng(seed)
    shapes = {"q": (HIDDEN, HIDDEN), "k": (HIDDEN, HIDDEN), "v": (HIDDEN, HIDDEN), "o": (HIDDEN, HIDDEN),
              "gate": (INTER, HIDDEN), "up": (INTER, HIDDEN), "down": (HIDDEN, INTER)}
    W = {n: rng.standard_normal(s) * 0.3 for n, s in shapes.items()}
    A = {n: rng.standard_normal((CFG["r"], s[1])) * 0.5 for n, s in shapes.items()}
    B = {n: rng.standard_normal((s[0], CFG["r"])) * 0.5 for n, s in shapes.items()}
    g1 = 1.0 + 0.2 * rng.standard_normal(HIDDEN)
    g2 = 1.0 + 0.2 * rng.standard_normal(HIDDEN)
    x = rng.standard_normal((CFG["batch"] * CFG["seq"], HIDDEN))
    dy = rng.standard_normal(x.shape)
    return x, W, A, B, g1, g2, dy


def test_block_backward_against_finite_differences():
    x, W, A, B, g1, g2, dy = _params(1)
    dx, dA, dB = block.backward(x, CFG, W, A, B, g1, g2, dy)

    def loss(x_=x, A_=A, B_=B):
        return float(np.sum(dy * block.forward(x_, CFG, W, A_, B_, g1, g2)))

    h = 1e-6
    for idx in np.ndindex(x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        fd = (loss(x_=xp) - loss(x_=xm)) / (2 * h)
        assert abs(fd - dx[idx]) <= 1e-6 * max(1.0, abs(fd)), ("x", idx)
    rng = np.random.default_rng(2)
    for n in block.NAMES:
        for which, P, G in (("A", A, dA), ("B", B, dB)):
            for _ in range(4):
                idx = tuple(rng.integers(0, d) for d in P[n].shape)
                Pp = {k: v.copy() for k, v in P.items()}
                Pm = {k: v.copy() for k, v in P.items()}
                Pp[n][idx] += h
                Pm[n][idx] -= h
                kw_p = {"A_": Pp} if which == "A" else {"B_": Pp}
                kw_m = {"A_": Pm} if which == "A" else {"B_": Pm}
                fd = (loss(**kw_p) - loss(**kw_m)) / (2 * h)
                assert abs(fd - G[n][idx]) <= 1e-6 * max(1.0, abs(fd)), (which, n, idx)


def test_rmsnorm_of_a_constant_row_is_the_weight():
    g = np.array([0.5, 2.0, -1.0, 3.0])
    u, rstd = block.rmsnorm(np.full((1, 4), -2.5), g, eps=0.0)
    np.testing.assert_allclose(u[0], -g, rtol=1e-15)
    assert rstd[0] == 1 / 2.5


def test_rope_is_a_rotation_and_identity_at_position_zero():
    rng = np.random.default_rng(3)
    b, s, H, D = 2, 6, 3, 8
    t = rng.standard_normal((b * s, H * D))
    r = block.rope(t, b, s, H, D, 10000.0)
    rr = r.reshape(b, s, H, D)
    tt = t.reshape(b, s, H, D)
    np.testing.assert_array_equal(rr[:, 0], tt[:, 0])                   # angle 0
    np.testing.assert_allclose(np.linalg.norm(rr, axis=-1), np.linalg.norm(tt, axis=-1), rtol=1e-13)
    np.testing.assert_allclose(block.rope(r, b, s, H, D, 10000.0, inverse=True), t, atol=1e-13)
    # one pair by hand: position 3, pair 0 of head 1 rotates by 3 * base^0 = 3 rad
    a, c = tt[1, 3, 1, 0], tt[1, 3, 1, D // 2]
    assert abs(rr[1, 3, 1, 0] - (a * np.cos(3.0) - c * np.sin(3.0))) < 1e-13
    assert abs(rr[1, 3, 1, D // 2] - (a * np.sin(3.0) + c * np.cos(3.0))) < 1e-13


def test_attention_closed_forms():
    rng = np.random.default_rng(4)
    H, D = 2, 4
    v = rng.standard_normal((3, H * D))
    q = rng.standard_normal((3, H * D))
    # one token per sequence: the output is v
    a, _ = block.attention(q, rng.standard_normal((3, H * D)), v, 3, 1, H, D)
    np.testing.assert_allclose(a, v, rtol=1e-15)
    # identical keys: uniform weights over the causal prefix
    k = np.tile(rng.standard_normal((1, H * D)), (3, 1))
    a, _ = block.attention(q, k, v, 1, 3, H, D)
    want = np.cumsum(v, axis=0) / np.arange(1, 4)[:, None]
    np.testing.assert_allclose(a, want, rtol=1e-13)


def test_silu_closed_forms():
    """silu(z) = z * sigmoid(z): sigmoid(ln 3) = 3/4 exactly, silu(0) = 0, and
    silu(z) - silu(-z) = z for every z (sigmoid(z) + sigmoid(-z) = 1)."""
    ln3 = np.log(3.0)
    np.testing.assert_allclose(block.silu(np.array([ln3, -ln3, 0.0])), [0.75 * ln3, -0.25 * ln3, 0.0], rtol=1e-15)
    z = np.linspace(-20, 20, 81)
    np.testing.assert_allclose(block.silu(z) - block.silu(-z), z, rtol=1e-14, atol=1e-14)
