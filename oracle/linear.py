"""QLoRA linear layer, forward and backward, in float64 (oracle side).

TEST INFRASTRUCTURE (see the package docstring).

The layer (mbrenndoerfer.com QLoRA essay, section "Low-Rank Adaptation
(LoRA)": x_out = (W_q + BA) x_in, with A of shape r x d and B of shape d x r;
"QLoRA: Efficient Finetuning of Quantized LLMs", section "Method": the 4-bit
weight is dequantized to BFloat16 and used in a 16-bit matrix multiplication;
gradients are backpropagated through the frozen quantized weight into the
adapters only, so there is no gradient for W).

Row-vector convention, as in nn.Linear:
  X  [M, K]  tokens x in_features          W' [N, K] dequantized weight (bf16)
  A  [r, K]  B [N, r]  s = lora_alpha / r (the usual LoRA scale; the pages
  print alpha and r but no formula)
  Y  = X W'^T + s (X A^T) B^T
and with dY = dL/dY:
  dX = dY W' + s (dY B) A
  dA = s (dY B)^T X
  dB = s dY^T (X A^T)
Every operand is exactly the bf16 (or float32) value handed to the GPU,
widened to float64; numpy's float64 matmul is the only library step.
"""

import numpy as np


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def forward(X, Wd, A, B, s: float) -> np.ndarray:
    X, Wd, A, B = map(_f64, (X, Wd, A, B))
    return X @ Wd.T + s * ((X @ A.T) @ B.T)


def backward(X, Wd, A, B, s: float, dY):
    """(dX, dA, dB)."""
    X, Wd, A, B, dY = map(_f64, (X, Wd, A, B, dY))
    G = dY @ B                     # [M, r]
    dX = dY @ Wd + s * (G @ A)
    dA = s * (G.T @ X)
    dB = s * (dY.T @ (X @ A.T))
    return dX, dA, dB


def forward_rows(X, Wd, A, B, s: float, rows) -> np.ndarray:
    """Forward restricted to the token rows `rows` (for spot checks at sizes
    where the whole product would be slow on the CPU)."""
    return forward(_f64(X)[rows], Wd, A, B, s)


def backward_dx_rows(Wd, A, B, s: float, dY, rows) -> np.ndarray:
    dYr = _f64(dY)[rows]
    Wd, A, B = map(_f64, (Wd, A, B))
    return dYr @ Wd + s * ((dYr @ B) @ A)


def backward_weight_grads(X, A, B, s: float, dY):
    """(dA, dB) alone, the same products as backward() without the input
    gradient (whose dY W' term dominates the cost at LLaMA sizes)."""
    X, A, B, dY = map(_f64, (X, A, B, dY))
    G = dY @ B
    return s * (G.T @ X), s * (dY.T @ (X @ A.T))


# ---- LoRA dropout on the adapter input ------------------------------------------------
#
# The blog's LoraConfig snippet ("Efficient Language Model Fine-Tuning with
# QLoRA on Resource-Constrained Hardware", marciocunha.net) sets lora_dropout:
# the adapter branch sees X_d = X * mask / (1 - p) while the frozen base sees
# X.  With bf16 activations the dropped-out input is itself bf16: each kept
# element is RN_bf16(RN32(x * RN32(1 / (1 - p)))), each dropped one 0.  The
# gradient through the dropout is mask / (1 - p) (the rounding is a storage
# step, not part of the function being differentiated):
#   Y  = X W'^T + s (X_d A^T) B^T
#   dX = dY W' + (s (dY B) A) * mask / (1 - p)
#   dA = s (dY B)^T X_d,   dB = s dY^T (X_d A^T)

def dropout_scale(p: float) -> np.float32:
    """RN32(1 / RN32(1 - p)): one correctly rounded binary32 quotient (exact
    rational arithmetic, no intermediate rounding)."""
    from fractions import Fraction

    from . import exact
    keep = np.float32(np.float32(1.0) - np.float32(p))
    return exact.rn32(Fraction(1) / Fraction(float(keep)))


def dropout_input(X, mask, p: float, bf16_round=True) -> np.ndarray:
    """X_d: kept elements scaled by RN32(1/(1-p)) (and rounded to bf16), the
    others 0.  mask: bool [M, K], True = kept."""
    X = np.asarray(X, np.float32)
    sc = dropout_scale(p)
    v = (X * sc).astype(np.float32)
    if bf16_round:
        b = v.view(np.uint32).astype(np.uint64)
        b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000      # round to nearest even, to bf16
        v = b.astype(np.uint32).view(np.float32)
    return np.where(mask, v, np.float32(0.0)).astype(np.float64)


def forward_dropout(X, Wd, A, B, s: float, Xd) -> np.ndarray:
    X, Wd, A, B, Xd = map(_f64, (X, Wd, A, B, Xd))
    return X @ Wd.T + s * ((Xd @ A.T) @ B.T)


def backward_dropout(X, Wd, A, B, s: float, dY, Xd, mask, p: float):
    """(dX, dA, dB) of forward_dropout."""
    X, Wd, A, B, dY, Xd = map(_f64, (X, Wd, A, B, dY, Xd))
    G = dY @ B
    dX = dY @ Wd + s * (G @ A) * (np.asarray(mask, bool) * np.float64(dropout_scale(p)))
    return dX, s * (G.T @ Xd), s * (dY.T @ (Xd @ A.T))


def rel_frobenius(got, ref) -> float:
    got, ref = _f64(got), _f64(ref)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def max_abs(got, ref) -> float:
    return float(np.max(np.abs(_f64(got) - _f64(ref)))) if np.size(ref) else 0.0
