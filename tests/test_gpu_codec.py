"""GPU parity of the NF4 + double-quantization codec against the oracle.

"QLoRA: Efficient Finetuning of Quantized LLMs", section "Method": NF4
quantization with blocksize 64 (step (3) of "4-bit NormalFloat
Quantization"), double quantization of the block constants, dequantization to
BFloat16.  Packed codes, E4M3 codes, scales, mean and the dequantized bf16
weight must match the oracle bit for bit.
"""

import numpy as np
import pytest
import torch

import synthetic
from oracle import codebook as ocb
from oracle import codec as occ

pytestmark = pytest.mark.gpu

Q = ocb.nf4_codebook()


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_16_b200 as q
    assert torch.cuda.is_available()
    return q


def gpu_quantize(q, W: torch.Tensor, codebook=None):
    rows, cols = W.shape
    w = q.NF4Weight(rows, cols, codebook=codebook, device="cuda")
    ws = torch.empty(q.qlora_quantize_workspace_bytes(rows, cols), dtype=torch.uint8, device="cuda")
    q.qlora_quantize_nf4_dq(W.cuda().contiguous(), w, ws)
    torch.cuda.synchronize()
    return w


def gpu_dequantize(q, w):
    out = torch.empty(w.rows, w.cols, dtype=torch.bfloat16, device="cuda")
    q.qlora_dequantize_nf4_dq(w, out)
    torch.cuda.synchronize()
    return out.view(torch.int16).cpu().numpy().view(np.uint16).ravel()


def check_parity(q, W: torch.Tensor, codebook=None):
    table = Q if codebook is None else np.asarray(codebook, np.float32)
    w = gpu_quantize(q, W, codebook)
    ref = occ.quantize(W.float().numpy(), table)
    assert np.array_equal(w.packed.cpu().numpy(), ref["packed"]), "packed codes"
    assert np.array_equal(w.code2.cpu().numpy(), ref["e"]), "E4M3 codes"
    assert np.array_equal(w.c2.cpu().numpy().view(np.uint32), ref["c2"].view(np.uint32)), "group scales"
    assert w.mean[0].item() == float(ref["mean"]), "mean"
    got = gpu_dequantize(q, w)
    want = occ.dequantize(ref["packed"], ref["e"], ref["c2"], ref["mean"], table)
    assert np.array_equal(got, want), "dequantized bf16"
    return w, ref


def test_codebook_in_weight_descriptor_is_the_oracle_table(q):
    assert np.array_equal(np.array(q.qlora_build_nf4_codebook(), np.float32).view(np.uint32), Q.view(np.uint32))


def test_tiny_config_fp32(q):
    case = synthetic.tiny_linear(seed=0)
    check_parity(q, case["W"])


@pytest.mark.parametrize("rows,cols", [(1, 64), (3, 192), (100, 192), (257, 320), (512, 1024)])
def test_ragged_shapes_bf16(q, rows, cols):
    check_parity(q, synthetic.normal((rows, cols), 0.02, seed=rows + cols, dtype=torch.bfloat16))


def test_llama_7b_shapes_bf16(q):
    for i, (rows, cols) in enumerate([(4096, 4096), (11008, 4096), (4096, 11008)]):
        check_parity(q, synthetic.normal((rows, cols), 0.02, seed=40 + i, dtype=torch.bfloat16))


def test_llama_65b_shapes_bf16(q):
    """The largest tensors of the 65B configurations, compared in full: 8192²
    (attention) and 22016 x 8192 (2.8 M blocks, about 25 warp-steps per warp)."""
    for i, (rows, cols) in enumerate([(8192, 8192), (22016, 8192)]):
        check_parity(q, synthetic.normal((rows, cols), 0.02, seed=60 + i, dtype=torch.bfloat16))


def test_int4_codebook(q):
    """The Int4 table through the same quantizer and dequantizer: ragged and
    full-size tensors, a zero block (the table's zero is index 8) and exact
    midpoints."""
    table = q.qlora_build_int4_codebook()
    for i, (rows, cols) in enumerate([(3, 192), (257, 320), (4096, 4096)]):
        check_parity(q, synthetic.normal((rows, cols), 0.02, seed=80 + i, dtype=torch.bfloat16), table)
    W = synthetic.normal((4, 256), 0.02, seed=83)
    W[0, :64] = 0.0
    t = np.asarray(table, np.float64)
    mids = np.float32((t[1:] + t[:-1]) / 2)
    row = np.zeros(64, np.float32)
    row[0] = 1.0
    row[1:15] = mids[1:]
    row[15:29] = np.nextafter(mids[1:], np.float32(2))
    W[1, :64] = torch.from_numpy(row)
    w, ref = check_parity(q, W, table)
    assert np.all(occ.unpack(w.packed.cpu().numpy())[:64] == 8)


def test_fp4_codebook(q):
    """The 4-bit float (E2M1) table through the same quantizer and
    dequantizer: ragged and LLaMA-attention-shaped tensors, bit-exact."""
    table = q.qlora_build_fp4_codebook()
    assert np.array_equal(np.array(table, np.float32).view(np.uint32), ocb.fp4_codebook().view(np.uint32))
    for shape, seed in (((257, 320), 31), ((4096, 4096), 32)):
        W = synthetic.normal(shape, 0.02, seed, torch.bfloat16)
        w, ref = check_parity(q, W, codebook=table)
        codes = occ.unpack(ref["packed"])
        assert codes.min() >= 1, "index 0 (-8/6) is never the nearest value"


@pytest.mark.parametrize("k", [2, 3])
def test_nfk_codebooks(q, k):
    """NF3 and NF2 through the 4-bit quantizer and dequantizer, bit-exact;
    the padding codes beyond +-1 are never emitted."""
    table = q.qlora_build_nfk_codebook(k)
    W = synthetic.normal((300, 512), 0.02, 40 + k, torch.bfloat16)
    w, ref = check_parity(q, W, codebook=table)
    pad = (16 - 2 ** k) // 2
    codes = occ.unpack(ref["packed"])
    assert codes.min() >= pad and codes.max() < 16 - pad


def test_fp16_input_and_fp16_dequantization(q):
    """The fp16 compute dtype: fp16 weights quantize bit-exactly (the oracle
    reads them as the float32 values they are), and the dequantizer's fp16
    output is fp16_RNE(RN32(q * c1')) bit for bit."""
    for shape, seed in (((257, 320), 51), ((4096, 4096), 52)):
        W = synthetic.normal(shape, 0.02, seed, torch.float16)
        w, ref = check_parity(q, W)
        out = torch.empty(shape, dtype=torch.float16, device="cuda")
        q.qlora_dequantize_nf4_dq(w, out)
        torch.cuda.synchronize()
        got = out.view(torch.int16).cpu().numpy().view(np.uint16).ravel()
        want = occ.dequantize_f16(ref["packed"], ref["e"], ref["c2"], ref["mean"], Q)
        assert np.array_equal(got, want)


def test_edge_blocks(q):
    """Zero blocks, a subnormal block, values exactly on the round-down
    midpoints (ties go to the lower code), and +-absmax."""
    W = synthetic.normal((6, 256), 0.02, seed=7)
    W[0, :64] = 0.0
    W[1, :64] = -0.0
    W[1, 64:128] = 0.0
    W[1, 70] = 1e-40
    mids = []
    for j in range(15):
        m = np.float32((float(Q[j]) + float(Q[j + 1])) / 2)
        mids += [m, np.nextafter(m, np.float32(-2)), np.nextafter(m, np.float32(2))]
    row = np.zeros(64, np.float32)
    row[0] = 1.0
    row[1:1 + 45] = mids
    W[2, :64] = torch.from_numpy(row)
    W[3, :64] = -torch.from_numpy(row)
    check_parity(q, W)


def test_constant_tensor_has_zero_second_level(q):
    W = torch.full((8, 128), 0.03125, dtype=torch.bfloat16)
    w, ref = check_parity(q, W)
    assert np.all(ref["c2"] == 0) and np.all(ref["e"] == 0)


def test_exact_round_trip(q):
    rng = np.random.default_rng(9)
    a = np.float32(0.046875)
    codes = rng.integers(0, 16, (64, 256)).astype(np.uint8)
    codes[:, ::64] = rng.choice([0, 15], (64, 4))
    W = occ.bf16_bits_to_f32(occ.bf16_rne((Q[codes] * a).astype(np.float32)))
    w = gpu_quantize(q, torch.from_numpy(W).to(torch.bfloat16))
    got = gpu_dequantize(q, w)
    assert np.array_equal(got, torch.from_numpy(W).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).ravel())


def test_deterministic_bytes(q):
    W = synthetic.normal((1024, 4096), 0.02, seed=3, dtype=torch.bfloat16)
    a, b = gpu_quantize(q, W), gpu_quantize(q, W)
    for name in ("packed", "code2", "c2"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    assert a.mean[0].item() == b.mean[0].item()


def test_dequantize_of_oracle_encoded_weight(q):
    """The dequantizer alone, fed the oracle's quantized buffers."""
    W = synthetic.normal((300, 256), 0.02, seed=11).numpy()
    ref = occ.quantize(W, Q)
    w = q.NF4Weight(300, 256, device="cuda")
    w.packed.copy_(torch.from_numpy(ref["packed"]))
    w.code2.copy_(torch.from_numpy(ref["e"]))
    w.c2.copy_(torch.from_numpy(ref["c2"]))
    w.mean[0] = float(ref["mean"])
    got = gpu_dequantize(q, w)
    assert np.array_equal(got, occ.dequantize(ref["packed"], ref["e"], ref["c2"], ref["mean"], Q))


def test_bits_per_parameter_from_buffer_sizes(q):
    w = q.NF4Weight(4096, 4096, device="cuda")
    bits = 8 * w.nbytes / (4096 * 4096)
    assert bits == pytest.approx(occ.storage_bits_per_param(4096 * 4096), rel=1e-12)


def _blocks_with_absmax(c1: np.ndarray, seed: int) -> torch.Tensor:
    """fp32 weight [len(c1)/16, 1024] whose 64-blocks have exactly the given
    absmax values: element 0 of block b is c1[b], the others lie strictly
    inside (-c1[b], c1[b])."""
    rng = np.random.default_rng(seed)
    nb = len(c1)
    blocks = (rng.uniform(-0.9, 0.9, (nb, 64)) * c1[:, None]).astype(np.float32)
    blocks[:, 0] = c1
    return torch.from_numpy(blocks.reshape(nb // 16, 1024))


def _e4m3_midpoints():
    vals = sorted({occ.e4m3_value(c) for c in range(0x7F)} | {0.0})
    return [(a + b) / 2 for a, b in zip(vals, vals[1:])]


def test_double_quantization_on_e4m3_ties(q):
    """Block constants c1 = 1 +- t 2^-9 with t on every E4M3 rounding midpoint:
    the mean is exactly 1, every group's scale exactly 2^-9 (t = 448 is in
    each group), so (c1 - mean) / c2 = t is an exact tie that round-to-
    nearest-even must resolve (Double Quantization, E4M3 reading)."""
    mids = _e4m3_midpoints()
    groups = 32
    c1 = []
    for g in range(groups):
        ts = [448.0] + [mids[(127 * g + i) % len(mids)] for i in range(127)]
        for t in ts:
            c1 += [1.0 + t * 2.0 ** -9, 1.0 - t * 2.0 ** -9]
    c1 = np.array(c1, np.float32)
    assert c1.min() > 0 and len(c1) == 256 * groups
    w, ref = check_parity(q, _blocks_with_absmax(c1, 5))
    assert float(ref["mean"]) == 1.0 and np.all(ref["c2"] == np.float32(2.0 ** -9))


def test_double_quantization_near_e4m3_boundaries(q):
    """Group scale 3 2^-11 (its reciprocal is inexact) and quotients within a
    few float32 units of E4M3 rounding boundaries: the codes must equal the
    oracle's correctly rounded quotient everywhere."""
    mids = _e4m3_midpoints()
    c = 3.0 * 2.0 ** -11
    groups = 48
    c1 = []
    for g in range(groups):
        ts = [448.0]
        for i in range(127):
            m = mids[(5 * g + i) % len(mids)]
            ts.append(m * (1.0 + ((i % 7) - 3) * 2.0 ** -23))
        for t in ts:
            c1 += [1.0 + t * c, 1.0 - t * c]
    c1 = np.array(c1, np.float32)
    assert c1.min() > 0
    check_parity(q, _blocks_with_absmax(c1, 6))


def test_back_to_back_calls_share_one_workspace(q):
    """Several quantize calls queued on one stream with one workspace and no
    host synchronization between them: each call resets the shared reduction
    slots and arrival ticket only after the call before it has finished with
    them, so every weight matches the oracle."""
    shapes = [(4096, 4096), (64, 4096), (11008, 4096), (3, 192), (4096, 11008)]
    Ws = [synthetic.normal(s, 0.02, seed=90 + i, dtype=torch.bfloat16) for i, s in enumerate(shapes)]
    nbytes = max(q.qlora_quantize_workspace_bytes(r, c) for r, c in shapes)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    Wd = [W.cuda() for W in Ws]
    outs = [q.NF4Weight(r, c, device="cuda") for r, c in shapes]
    torch.cuda.synchronize()
    for W, w in zip(Wd, outs):
        q.qlora_quantize_nf4_dq(W, w, ws)
    torch.cuda.synchronize()
    for W, w in zip(Ws, outs):
        ref = occ.quantize(W.float().numpy(), Q)
        assert np.array_equal(w.packed.cpu().numpy(), ref["packed"]), "packed codes"
        assert np.array_equal(w.code2.cpu().numpy(), ref["e"]), "E4M3 codes"
        assert np.array_equal(w.c2.cpu().numpy().view(np.uint32), ref["c2"].view(np.uint32)), "group scales"
        assert w.mean[0].item() == float(ref["mean"]), "mean"
