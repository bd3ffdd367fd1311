"""GPU parity of the paged optimizer's AdamW update against the float64 oracle.

"QLoRA: Efficient Finetuning of Quantized LLMs", Introduction item (3) and
section "Method": paged optimizers keep the optimizer states in NVIDIA unified
memory; they are evicted to CPU RAM under memory pressure and paged back for
the update.  The update is AdamW (the oracle's docstring gives the reading).

Tolerance, from the float32 arithmetic of the kernel: each step rounds about
eight times (decay, the two moment updates, square root, two divisions, the
step-size product and the subtraction), and the float32 step scalars carry one
rounding each; errors in m and v carry over from step to step.  After T steps
the parameters are within 64 * T units of 2^-24 of (|p| + lr) of the exact
result, m within 16 * T * 2^-24 * max|g| and v within 16 * T * 2^-24 * max g^2.
"""

import numpy as np
import pytest
import torch

import synthetic
from oracle import optim as oopt

pytestmark = pytest.mark.gpu

HP = dict(lr=2e-3, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.01)
U = 2.0 ** -24


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_16_b200 as q
    assert torch.cuda.is_available()
    return q


def grads_for(n, steps, seed):
    return [synthetic.normal((n,), 1e-3, seed + t) for t in range(steps)]


def run(q, n, steps, paged, evict=False, seed=40):
    p0 = synthetic.normal((n,), 0.02, seed - 1)
    p = p0.cuda()
    p16 = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    bufs = None
    if paged:
        bufs = (q.PagedBuffer(n), q.PagedBuffer(n))
        m, v = bufs[0].tensor, bufs[1].tensor
    else:
        m = torch.zeros(n, dtype=torch.float32, device="cuda")
        v = torch.zeros(n, dtype=torch.float32, device="cuda")
    for t, g in enumerate(grads_for(n, steps, seed), start=1):
        if evict:
            for b in bufs:
                q.qlora_paged_prefetch(b, to_device=False)
        q.qlora_adamw_step(p, p16, g.cuda(), m, v, HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["wd"], t)
    q.qlora_check_device_error()
    out = (p.cpu(), p16.cpu(), m.cpu().clone(), v.cpu().clone())
    if bufs:
        for b in bufs:
            b.free()
    return p0, out


@pytest.mark.parametrize("n", [4096, 10007])   # whole float4 groups; a 3-element tail
def test_adamw_matches_oracle(q, n):
    steps = 5
    p0, (p, p16, m, v) = run(q, n, steps, paged=False)
    grads = [g.numpy() for g in grads_for(n, steps, 40)]
    rp, rm, rv = oopt.adamw(p0.numpy(), grads, **HP)
    gmax = max(np.abs(g).max() for g in grads)
    T = steps
    assert np.all(np.abs(p.numpy() - rp) <= 64 * T * U * (np.abs(rp) + HP["lr"]))
    assert np.all(np.abs(m.numpy() - rm) <= 16 * T * U * gmax)
    assert np.all(np.abs(v.numpy() - rv) <= 16 * T * U * gmax ** 2)
    # the bf16 copy is the round-to-nearest-even of the float32 parameters
    assert torch.equal(p16, p.to(torch.bfloat16))


def test_paged_state_gives_identical_bits(q):
    """m and v in unified memory, evicted to the host before every step (the
    update pages them back on demand): the same bits as device memory."""
    n = 65539
    _, dev = run(q, n, 4, paged=False, seed=70)
    _, pg = run(q, n, 4, paged=True, evict=True, seed=70)
    for a, b in zip(dev, pg):
        assert torch.equal(a, b)


def test_adamw_argument_errors(q):
    p = torch.zeros(16, device="cuda")
    g = torch.zeros(16, device="cuda")
    m = torch.zeros(16, device="cuda")
    v = torch.zeros(16, device="cuda")
    for kw, status in ((dict(step=0), 1), (dict(beta1=1.0), 1), (dict(eps=0.0), 1), (dict(lr=-1.0), 1)):
        a = dict(HP, step=1)
        a.update(kw)
        with pytest.raises(q.QLoraError) as e:
            q.qlora_adamw_step(p, None, g, m, v, a["lr"], a["beta1"], a["beta2"], a["eps"], a["wd"], a["step"])
        assert e.value.status == status
    with pytest.raises(q.QLoraError) as e:
        q.qlora_adamw_step(p[1:], None, g[1:], m[1:], v[1:], HP["lr"], HP["beta1"], HP["beta2"], HP["eps"],
                           HP["wd"], 1)
    assert e.value.status == 3
