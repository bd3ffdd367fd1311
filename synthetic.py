"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

Holds no arithmetic of the method: only random tensors with the shapes and
distributions of the workloads (normally distributed weights, as the QLoRA
paper's section "Method" assumes for pretrained weights, and N(0, 1)
activations and output gradients).  Both the CUDA path and the oracle receive
exactly these tensors.

Notation: N(0, s) below means standard deviation s.
"""

import torch

# LLaMA-7B projection shapes (out_features N, in_features K): q/k/v/o, gate/up, down
LLAMA7B_LINEARS = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                   ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
LLAMA7B_LAYERS = 32
# LLaMA-65B projection shapes
LLAMA65B_LINEARS = [("q", 8192, 8192), ("k", 8192, 8192), ("v", 8192, 8192), ("o", 8192, 8192),
                    ("gate", 22016, 8192), ("up", 22016, 8192), ("down", 8192, 22016)]
LLAMA65B_LAYERS = 80


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(shape, std: float, seed: int, dtype=torch.float32, device="cpu") -> torch.Tensor:
    """N(0, std) tensor drawn in float32 from a seeded generator, then cast."""
    t = torch.randn(*shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return (t * std).to(dtype)


def tiny_linear(seed: int = 0, device="cpu") -> dict:
    """The tiny QLoRA linear: W 256x256 fp32 N(0, 0.02); X 16x256 bf16 N(0, 1);
    r = 8, alpha = 16; A N(0, 1/r); B N(0, 0.01); dY N(0, 1)."""
    return linear_case(M=16, N=256, K=256, r=8, alpha=16.0, seed=seed, w_dtype=torch.float32, device=device)


def linear_case(M: int, N: int, K: int, r: int, alpha: float, seed: int, w_dtype=torch.bfloat16,
                device="cpu", act_dtype=torch.bfloat16) -> dict:
    """One QLoRA linear problem with the workload's distributions (act_dtype:
    the 16-bit compute dtype of X, A, B and dY)."""
    return {
        "W": normal((N, K), 0.02, seed, w_dtype, device),
        "X": normal((M, K), 1.0, seed + 1, act_dtype, device),
        "A": normal((r, K), 1.0 / r, seed + 2, act_dtype, device),
        "B": normal((N, r), 0.01, seed + 3, act_dtype, device),
        "dY": normal((M, N), 1.0, seed + 4, act_dtype, device),
        "r": r, "alpha": alpha, "scale": alpha / r, "M": M, "N": N, "K": K,
    }


def block_case(batch: int, seq: int, hidden: int, heads: int, inter: int, r: int, alpha: float, seed: int,
               device="cpu") -> dict:
    """One transformer block problem: the seven weights N(0, 0.02) in the
    shapes (out, in) of q, k, v, o (hidden x hidden), gate, up (inter x
    hidden), down (hidden x inter); adapters A N(0, 1/r), B N(0, 0.01); norm
    weights 1 + N(0, 0.1); block input x and output gradient dy N(0, 1)."""
    shapes = [(hidden, hidden)] * 4 + [(inter, hidden)] * 2 + [(hidden, inter)]
    W = [normal(s, 0.02, seed + 10 * i, torch.bfloat16, device) for i, s in enumerate(shapes)]
    A = [normal((r, s[1]), 1.0 / r, seed + 10 * i + 1, torch.bfloat16, device) for i, s in enumerate(shapes)]
    B = [normal((s[0], r), 0.01, seed + 10 * i + 2, torch.bfloat16, device) for i, s in enumerate(shapes)]
    T = batch * seq
    return {
        "W": W, "A": A, "B": B,
        "norm1": (1.0 + normal((hidden,), 0.1, seed + 101)).to(torch.bfloat16).to(device),
        "norm2": (1.0 + normal((hidden,), 0.1, seed + 102)).to(torch.bfloat16).to(device),
        "x": normal((T, hidden), 1.0, seed + 103, torch.bfloat16, device),
        "dy": normal((T, hidden), 1.0, seed + 104, torch.bfloat16, device),
        "batch": batch, "seq": seq, "hidden": hidden, "heads": heads, "inter": inter, "r": r,
        "alpha": alpha, "scale": alpha / r,
    }


def dropout_mask(M: int, K: int, p: float, seed: int, device="cpu"):
    """LoRA-dropout keep mask: (bool [M, K] with P(kept) = 1 - p, and the same
    mask packed 8 elements per byte, bit k % 8 of byte (m*K + k) / 8)."""
    g = _gen(seed)
    keep = torch.rand(M, K, generator=g) >= p
    bits = keep.reshape(-1, 8).to(torch.uint8)
    weights = torch.tensor([1, 2, 4, 8, 16, 32, 64, 128], dtype=torch.uint8)
    packed = (bits * weights).sum(dim=1).to(torch.uint8)
    return keep, packed.to(device)
