"""GPU parity of the QLoRA transformer block (forward, and backward with
gradient checkpointing) against the float64 oracle.

"QLoRA: Efficient Finetuning of Quantized LLMs", Introduction: adapters at
every layer, gradient checkpointing; the LLaMA block layout is the reading
stated in oracle/block.py.  The oracle runs on the GPU's own quantized
weights (dequantized by the oracle codec) and on the same bf16 inputs.

Tolerance, from the arithmetic: the GPU stores every activation between
kernels in bf16 (each store rounds by at most 2^-9 relative), the oracle keeps
all of them exact.  The longest path from x to y passes 12 such stores (u1,
q/k/v, RoPE, P, a, o, h, u2, gate/up, m, down, y), so an element is within
12 * 2^-9 (2.3%) of the exact value relative to the magnitudes it was formed
from; the bar is relative Frobenius error <= 3e-2 and every element within
3e-2 of the tensor's largest reference magnitude.  The same bar holds for dx
and the adapter gradients, whose paths are of the same length.
"""

import numpy as np
import pytest
import torch

import synthetic
from oracle import block as oblk
from oracle import codebook as ocb
from oracle import codec as occ
from oracle import linear as olin

pytestmark = pytest.mark.gpu

Q = ocb.nf4_codebook()
REL = 3e-2


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_16_b200 as q
    assert torch.cuda.is_available()
    return q


def np64(t):
    return t.float().cpu().numpy().astype(np.float64)


def close(got, ref, what):
    got, ref = np64(got) if torch.is_tensor(got) else got, np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), what
    rel = olin.rel_frobenius(got, ref)
    scale = np.abs(ref).max()
    err = np.abs(got - ref).max()
    assert rel <= REL, f"{what}: rel Frobenius {rel:.3e}"
    assert err <= REL * scale, f"{what}: max abs {err:.3e} vs scale {scale:.3e}"
    return rel


def build(q, case):
    weights = []
    for W in case["W"]:
        w = q.NF4Weight(*W.shape)
        ws = torch.empty(q.qlora_quantize_workspace_bytes(*W.shape), dtype=torch.uint8, device="cuda")
        q.qlora_quantize_nf4_dq(W.cuda(), w, ws)
        weights.append(w)
    A = [a.cuda() for a in case["A"]]
    B = [b.cuda() for b in case["B"]]
    blk = q.Block(case["batch"], case["seq"], case["hidden"], case["heads"], case["inter"], case["r"],
                  case["scale"], weights, A, B, case["norm1"].cuda(), case["norm2"].cuda())
    blk._keep = (A, B)
    return blk


def oracle_inputs(case):
    Wd = {}
    for n, W in zip(oblk.NAMES, case["W"]):
        ref = occ.quantize(W.float().numpy(), Q)
        Wd[n] = occ.bf16_bits_to_f32(occ.dequantize(ref["packed"], ref["e"], ref["c2"], ref["mean"], Q)).reshape(
            W.shape).astype(np.float64)
    A = {n: np64(a) for n, a in zip(oblk.NAMES, case["A"])}
    B = {n: np64(b) for n, b in zip(oblk.NAMES, case["B"])}
    cfg = dict(batch=case["batch"], seq=case["seq"], heads=case["heads"], head_dim=case["hidden"] // case["heads"],
               r=case["r"], scale=case["scale"], eps=1e-6, rope_base=10000.0)
    return cfg, Wd, A, B, np64(case["norm1"]), np64(case["norm2"])


def run_case(q, case):
    blk = build(q, case)
    T, d = case["batch"] * case["seq"], case["hidden"]
    ws = torch.empty(q.qlora_block_workspace_bytes(blk), dtype=torch.uint8, device="cuda")
    x, dy = case["x"].cuda(), case["dy"].cuda()
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    q.qlora_block_fwd(blk, x, y, ws)
    dx = torch.empty_like(y)
    dA = [torch.empty(case["r"], W.shape[1], dtype=torch.float32, device="cuda") for W in case["W"]]
    dB = [torch.empty(W.shape[0], case["r"], dtype=torch.float32, device="cuda") for W in case["W"]]
    q.qlora_block_bwd(blk, x, dy, dx, dA, dB, ws)
    q.qlora_check_device_error()

    cfg, Wd, A, B, g1, g2 = oracle_inputs(case)
    xn, dyn = np64(case["x"]), np64(case["dy"])
    ry = oblk.forward(xn, cfg, Wd, A, B, g1, g2)
    rdx, rdA, rdB = oblk.backward(xn, cfg, Wd, A, B, g1, g2, dyn)
    rels = {"y": close(y, ry, "y"), "dx": close(dx, rdx, "dx")}
    for i, n in enumerate(oblk.NAMES):
        rels["dA_" + n] = close(dA[i], rdA[n], f"dA[{n}]")
        rels["dB_" + n] = close(dB[i], rdB[n], f"dB[{n}]")
    print({k: f"{v:.2e}" for k, v in rels.items()})
    return y, dx, dA, dB


def test_tiny_block(q):
    """32 tokens (2 sequences of 16), hidden 256 in two heads of 128."""
    run_case(q, synthetic.block_case(2, 16, 256, 2, 512, 16, alpha=16.0, seed=2000))


def test_mid_block_deterministic(q):
    """256 tokens (2 x 128), hidden 1024 in eight heads; a second backward
    pass gives the same bits."""
    case = synthetic.block_case(2, 128, 1024, 8, 2816, 64, alpha=16.0, seed=2100)
    y, dx, dA, dB = run_case(q, case)
    blk = build(q, case)
    ws = torch.empty(q.qlora_block_workspace_bytes(blk), dtype=torch.uint8, device="cuda")
    dx2 = torch.empty_like(dx)
    dA2 = [torch.empty_like(t) for t in dA]
    dB2 = [torch.empty_like(t) for t in dB]
    q.qlora_block_bwd(blk, case["x"].cuda(), case["dy"].cuda(), dx2, dA2, dB2, ws)
    assert torch.equal(dx, dx2) and all(torch.equal(a, b) for a, b in zip(dA + dB, dA2 + dB2))


def test_llama7b_block(q):
    """A LLaMA-7B block (hidden 4096, 32 heads of 128, inter 11008, r = 64) on
    one sequence of 512 tokens."""
    run_case(q, synthetic.block_case(1, 512, 4096, 32, 11008, 64, alpha=16.0, seed=2200))


def test_block_argument_errors(q):
    case = synthetic.block_case(1, 16, 256, 2, 512, 16, alpha=16.0, seed=2300)
    blk = build(q, case)
    ws = torch.empty(q.qlora_block_workspace_bytes(blk), dtype=torch.uint8, device="cuda")
    x = case["x"].cuda()
    y = torch.empty_like(x)
    with pytest.raises(q.QLoraError) as e:
        q.qlora_block_fwd(blk, x, y, ws[:1024])
    assert e.value.status == 4
    blk.desc.heads = 3   # heads * head_dim != hidden
    with pytest.raises(q.QLoraError) as e:
        q.qlora_block_fwd(blk, x, y, ws)
    assert e.value.status == 2
