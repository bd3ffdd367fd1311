"""AdamW in float64 (oracle side) for the paged optimizer.

TEST INFRASTRUCTURE (see the package docstring).

"QLoRA: Efficient Finetuning of Quantized LLMs", Introduction item (3) and
section "Method": paged optimizers keep the optimizer states in unified memory
so that they can be evicted to CPU RAM and paged back for the update.  The
pages name no optimizer; the reading is Adam with decoupled weight decay
(Loshchilov and Hutter, "Decoupled Weight Decay Regularization", the AdamW
algorithm): with t counting from 1,
    m_t = b1 m_{t-1} + (1 - b1) g_t
    v_t = b2 v_{t-1} + (1 - b2) g_t^2
    mhat = m_t / (1 - b1^t),  vhat = v_t / (1 - b2^t)
    p_t = p_{t-1} - lr (mhat / (sqrt(vhat) + eps) + wd p_{t-1})
(the weight decay multiplied by the learning rate, as in common use).  Paging
moves the bytes of m and v, never their values, so it has no counterpart here.
"""

import numpy as np


def adamw_step(p, g, m, v, t: int, lr: float, beta1: float, beta2: float, eps: float, wd: float):
    """One step; returns (p, m, v) as new float64 arrays."""
    p, g, m, v = (np.asarray(a, np.float64) for a in (p, g, m, v))
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** t)
    vhat = v / (1.0 - beta2 ** t)
    p = p - lr * (mhat / (np.sqrt(vhat) + eps) + wd * p)
    return p, m, v


def adamw(p0, grads, lr: float, beta1: float, beta2: float, eps: float, wd: float):
    """Steps 1..len(grads) from zero moments; returns (p, m, v) after the last."""
    p = np.asarray(p0, np.float64)
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    for t, g in enumerate(grads, start=1):
        p, m, v = adamw_step(p, g, m, v, t, lr, beta1, beta2, eps, wd)
    return p, m, v
