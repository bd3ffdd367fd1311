"""GPU parity of the QLoRA forward for a handful of tokens (the decode shape,
1 <= M <= 16), which streams the packed weight through its own kernels,
against the float64 oracle.

Layer: x_out = (W_q + B A) x_in (mbrenndoerfer.com QLoRA essay, section
"Low-Rank Adaptation (LoRA)"), the 4-bit weight dequantized to BFloat16 and
used in a 16-bit matmul ("QLoRA: Efficient Finetuning of Quantized LLMs",
section "Method").  Tolerance as for the linear layer: relative Frobenius
error <= 5e-3 and max abs error <= 2e-2 (float32 outputs), widened by half a
bf16 unit in the last place for bf16 outputs.
"""

import numpy as np
import pytest
import torch

import synthetic
from oracle import linear as olin
from test_gpu_linear import Runner, assert_close, np64, oracle_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_16_b200 as q
    assert torch.cuda.is_available()
    return q


@pytest.mark.parametrize("M,N,K,r", [
    (1, 512, 1024, 64),      # one token
    (4, 264, 576, 8),        # rows not a multiple of 16, contraction ends on half a 128-wide step
    (9, 512, 512, 128),      # second 8-token tile, largest rank
    (16, 1024, 2048, 64),    # the largest token count on this path
    (3, 136, 320, 16),       # ragged everything
])
@pytest.mark.parametrize("ydt", [torch.float32, torch.bfloat16])
def test_decode_forward(q, M, N, K, r, ydt):
    case = synthetic.linear_case(M, N, K, r, alpha=16.0, seed=1000 + M + N + K + r)
    run = Runner(q, case)
    Wd = oracle_weight(case["W"])
    Y, H = run.fwd(ydt, save_h=True)
    X, A, B = (np64(case[k]) for k in ("X", "A", "B"))
    s = case["scale"]
    assert_close(np64(Y), olin.forward(X, Wd, A, B, s), bf16_out=ydt == torch.bfloat16, what="Y")
    np.testing.assert_allclose(np64(H), s * X @ A.T, rtol=1e-5, atol=1e-5)


def test_decode_deterministic_and_zero_adapter(q):
    case = synthetic.linear_case(16, 1024, 4096, 64, alpha=16.0, seed=77)
    run = Runner(q, case)
    y1, _ = run.fwd()
    y2, _ = run.fwd()
    assert torch.equal(y1, y2)
    case["B"] = torch.zeros_like(case["B"])
    run = Runner(q, case)
    Y, _ = run.fwd()
    assert_close(np64(Y), np64(case["X"]) @ oracle_weight(case["W"]).T, what="Y with B = 0")


def test_llama65b_decode_shapes(q):
    """The three LLaMA-65B linear shapes at decode token counts 1, 4 and 16,
    checked in full against the oracle (one quantized weight per shape)."""
    for i, (name, N, K) in enumerate([("q", 8192, 8192), ("gate", 22016, 8192), ("down", 8192, 22016)]):
        full = synthetic.linear_case(16, N, K, 64, alpha=16.0, seed=300 + i, device="cpu")
        Wd = oracle_weight(full["W"])
        run = Runner(q, full)
        A, B = np64(full["A"]), np64(full["B"])
        for M in (1, 4, 16):
            run.X = full["X"][:M].cuda().contiguous()
            run.M = M
            Y, _ = run.fwd()
            X = np64(full["X"][:M])
            assert_close(np64(Y), olin.forward(X, Wd, A, B, full["scale"]), what=f"{name} M={M} Y")
