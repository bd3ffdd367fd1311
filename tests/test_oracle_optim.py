"""Pins of the oracle's AdamW: the library routine it reduces to (torch's
AdamW in float64 on the CPU), the closed form of the first step, and the
pure-decay case.

"QLoRA: Efficient Finetuning of Quantized LLMs", Introduction item (3):
paged optimizers; the update itself is AdamW (Loshchilov and Hutter,
"Decoupled Weight Decay Regularization")."""

import numpy as np
import torch

from oracle import optim

HP = dict(lr=2e-3, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.01)


def test_matches_torch_adamw_float64():
    rng = np.random.default_rng(3)
    p0 = rng.standard_normal(257) * 0.02
    grads = [rng.standard_normal(257) * 1e-3 for _ in range(6)]
    p_ref, m_ref, v_ref = optim.adamw(p0, grads, **HP)
    t = torch.tensor(p0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([t], lr=HP["lr"], betas=(HP["beta1"], HP["beta2"]), eps=HP["eps"],
                            weight_decay=HP["wd"])
    for g in grads:
        t.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
    st = opt.state[t]
    np.testing.assert_allclose(t.detach().numpy(), p_ref, rtol=0, atol=1e-15)
    np.testing.assert_allclose(st["exp_avg"].numpy(), m_ref, rtol=1e-13, atol=0)
    np.testing.assert_allclose(st["exp_avg_sq"].numpy(), v_ref, rtol=1e-13, atol=0)


def test_first_step_closed_form():
    """With zero moments, mhat = g and vhat = g^2 after step 1."""
    rng = np.random.default_rng(4)
    p0, g = rng.standard_normal(64), rng.standard_normal(64)
    p1, m1, v1 = optim.adamw(p0, [g], **HP)
    want = p0 - HP["lr"] * (g / (np.abs(g) + HP["eps"]) + HP["wd"] * p0)
    np.testing.assert_allclose(p1, want, rtol=1e-14, atol=1e-16)
    np.testing.assert_allclose(m1, (1 - HP["beta1"]) * g, rtol=1e-15)
    np.testing.assert_allclose(v1, (1 - HP["beta2"]) * g * g, rtol=1e-15)


def test_zero_gradient_is_pure_decay():
    p0 = np.linspace(-1, 1, 9)
    p, m, v = optim.adamw(p0, [np.zeros(9)] * 5, **HP)
    np.testing.assert_allclose(p, p0 * (1 - HP["lr"] * HP["wd"]) ** 5, rtol=1e-15, atol=0)
    assert not m.any() and not v.any()
    p, _, _ = optim.adamw(p0, [np.zeros(9)] * 5, **dict(HP, wd=0.0))
    assert np.array_equal(p, p0)
