"""One QLoRA transformer block, forward and backward, in float64 (oracle side).

TEST INFRASTRUCTURE (see the package docstring).

"QLoRA: Efficient Finetuning of Quantized LLMs", Introduction: LoRA adapters
at every network layer, and gradient checkpointing, whose memory spikes the
paged optimizers absorb.  The pages fix the seven linear shapes of the
LLaMA models they finetune (q, k, v, o; gate, up; down) but not the rest of
the block.  Reading: the LLaMA decoder block,
    u1 = RMSNorm(x; g1)
    q, k, v = Lq(u1), Lk(u1), Lv(u1)                      (QLoRA linears)
    q, k = RoPE(q), RoPE(k)                                (per head)
    a = causal softmax(q k^T / sqrt(D)) v                  (per sequence, head)
    h = x + Lo(a)
    u2 = RMSNorm(h; g2)
    y = h + Ldown(silu(Lgate(u2)) * Lup(u2))
with RMSNorm(x; g) = x / sqrt(mean(x^2) + eps) * g and RoPE rotating the
pairs (i, i + D/2) of each head by the angle p * base^(-2i/D) at sequence
position p (the "rotate half" layout).  The norm weights and the quantized
weights are frozen: the backward pass returns dx and the adapter gradients.
Gradient checkpointing changes what is stored, not what is computed, so it
has no counterpart here.

Every linear is oracle.linear's QLoRA layer on the dequantized weight.
"""

import numpy as np

from . import linear

NAMES = ("q", "k", "v", "o", "gate", "up", "down")


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def rmsnorm(x, g, eps):
    x = _f64(x)
    rstd = 1.0 / np.sqrt(np.mean(x * x, axis=-1) + eps)
    return x * rstd[:, None] * _f64(g)[None, :], rstd


def rmsnorm_backward(x, g, eps, du):
    """dx of u = x * rstd * g for the output gradient du."""
    x, g, du = _f64(x), _f64(g), _f64(du)
    d = x.shape[-1]
    rstd = 1.0 / np.sqrt(np.mean(x * x, axis=-1) + eps)
    xhat = x * rstd[:, None]
    gdu = g[None, :] * du
    return rstd[:, None] * (gdu - xhat * (np.sum(gdu * xhat, axis=-1) / d)[:, None])


def rope_angles(seq, head_dim, base):
    half = head_dim // 2
    inv = base ** (-2.0 * np.arange(half) / head_dim)
    return np.arange(seq)[:, None] * inv[None, :]            # [seq, half]


def rope(t, batch, seq, heads, head_dim, base, inverse=False):
    """t [batch*seq, heads*head_dim]: rotate (i, i + D/2) of each head; the
    inverse rotation (the transpose) is the backward pass."""
    t = _f64(t).reshape(batch, seq, heads, head_dim)
    ang = rope_angles(seq, head_dim, base)
    c = np.cos(ang)[None, :, None, :]
    s = np.sin(ang)[None, :, None, :]
    if inverse:
        s = -s
    half = head_dim // 2
    a, b = t[..., :half], t[..., half:]
    out = np.concatenate([a * c - b * s, a * s + b * c], axis=-1)
    return out.reshape(batch * seq, heads * head_dim)


def _heads(t, batch, seq, heads, head_dim):
    return _f64(t).reshape(batch, seq, heads, head_dim).transpose(0, 2, 1, 3)   # [b, h, s, D]


def _merge(t):
    b, h, s, d = t.shape
    return t.transpose(0, 2, 1, 3).reshape(b * s, h * d)


def attention(q, k, v, batch, seq, heads, head_dim):
    """Causal softmax attention; returns (a, P) with P [b, h, s, s]."""
    Q, K, V = (_heads(t, batch, seq, heads, head_dim) for t in (q, k, v))
    S = Q @ K.transpose(0, 1, 3, 2) / np.sqrt(head_dim)
    S = np.where(np.tril(np.ones((seq, seq), bool))[None, None], S, -np.inf)
    S = S - S.max(axis=-1, keepdims=True)
    P = np.exp(S)
    P /= P.sum(axis=-1, keepdims=True)
    return _merge(P @ V), P


def attention_backward(q, k, v, P, da, batch, seq, heads, head_dim):
    Q, K, V, dA = (_heads(t, batch, seq, heads, head_dim) for t in (q, k, v, da))
    dV = P.transpose(0, 1, 3, 2) @ dA
    dP = dA @ V.transpose(0, 1, 3, 2)
    dS = P * (dP - np.sum(dP * P, axis=-1, keepdims=True)) / np.sqrt(head_dim)
    dQ = dS @ K
    dK = dS.transpose(0, 1, 3, 2) @ Q
    return _merge(dQ), _merge(dK), _merge(dV)


def silu(z):
    z = _f64(z)
    return z / (1.0 + np.exp(-z))


def forward(x, cfg, W, A, B, g1, g2, cache=None):
    """x [batch*seq, hidden]; W, A, B dicts keyed by NAMES (W dequantized).
    cfg: batch, seq, heads, head_dim, r, scale, eps, rope_base."""
    b, s, H, D = cfg["batch"], cfg["seq"], cfg["heads"], cfg["head_dim"]
    sc = cfg["scale"]
    lin = lambda n, inp: linear.forward(inp, W[n], A[n], B[n], sc)
    u1, _ = rmsnorm(x, g1, cfg["eps"])
    q0, k0, v = lin("q", u1), lin("k", u1), lin("v", u1)
    q = rope(q0, b, s, H, D, cfg["rope_base"])
    k = rope(k0, b, s, H, D, cfg["rope_base"])
    a, P = attention(q, k, v, b, s, H, D)
    h = _f64(x) + lin("o", a)
    u2, _ = rmsnorm(h, g2, cfg["eps"])
    gt, up = lin("gate", u2), lin("up", u2)
    m = silu(gt) * up
    y = h + lin("down", m)
    if cache is not None:
        cache.update(u1=u1, q=q, k=k, v=v, P=P, a=a, h=h, u2=u2, gt=gt, up=up, m=m)
    return y


def backward(x, cfg, W, A, B, g1, g2, dy):
    """(dx, dA, dB) with dA, dB dicts keyed by NAMES."""
    b, s, H, D = cfg["batch"], cfg["seq"], cfg["heads"], cfg["head_dim"]
    sc = cfg["scale"]
    c = {}
    forward(x, cfg, W, A, B, g1, g2, cache=c)
    dA, dB = {}, {}

    def lin_bwd(n, inp, dout):
        dX, dA[n], dB[n] = linear.backward(inp, W[n], A[n], B[n], sc, dout)
        return dX

    dy = _f64(dy)
    dm = lin_bwd("down", c["m"], dy)
    sg = silu(c["gt"])
    sig = 1.0 / (1.0 + np.exp(-c["gt"]))
    dgt = dm * c["up"] * (sig + c["gt"] * sig * (1.0 - sig))
    dup = dm * sg
    du2 = lin_bwd("gate", c["u2"], dgt) + lin_bwd("up", c["u2"], dup)
    dh = dy + rmsnorm_backward(c["h"], g2, cfg["eps"], du2)
    da = lin_bwd("o", c["a"], dh)
    dq, dk, dv = attention_backward(c["q"], c["k"], c["v"], c["P"], da, b, s, H, D)
    dq0 = rope(dq, b, s, H, D, cfg["rope_base"], inverse=True)
    dk0 = rope(dk, b, s, H, D, cfg["rope_base"], inverse=True)
    du1 = lin_bwd("q", c["u1"], dq0) + lin_bwd("k", c["u1"], dk0) + lin_bwd("v", c["u1"], dv)
    dx = dh + rmsnorm_backward(x, g1, cfg["eps"], du1)
    return dx, dA, dB
