"""GPU parity of the QLoRA linear layer (forward and backward) against the
float64 oracle.

Layer: x_out = (W_q + B A) x_in (mbrenndoerfer.com QLoRA essay, section
"Low-Rank Adaptation (LoRA)"), with the 4-bit weight dequantized to BFloat16
and used in a 16-bit matmul ("QLoRA: Efficient Finetuning of Quantized LLMs",
section "Method"); gradients reach only the adapters (abstract).

Tolerance: relative Frobenius error <= 5e-3 and max abs error <= 2e-2 for
float32 outputs (fp32 accumulation).  For bf16 outputs the max-abs bound is
widened by half a bf16 unit in the last place of the reference value, the
rounding of the output itself.
"""

import numpy as np
import pytest
import torch

import synthetic
from oracle import codebook as ocb
from oracle import codec as occ
from oracle import linear as olin

pytestmark = pytest.mark.gpu

Q = ocb.nf4_codebook()
REL_FRO = 5e-3
MAX_ABS = 2e-2


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_16_b200 as q
    assert torch.cuda.is_available()
    return q


def half_ulp_bf16(ref):
    a = np.abs(np.asarray(ref, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 8)


def half_ulp_f16(ref):
    a = np.abs(np.asarray(ref, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return 2.0 ** (e - 11)


def assert_close(got, ref, bf16_out=False, what="", f16_out=False):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, what
    assert np.all(np.isfinite(got)), what
    rel = olin.rel_frobenius(got, ref)
    assert rel <= REL_FRO, f"{what}: rel Frobenius {rel:.3e}"
    bound = MAX_ABS + (half_ulp_bf16(ref) if bf16_out else 0.0) + (half_ulp_f16(ref) if f16_out else 0.0)
    err = np.abs(got - ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape) if err.size else None
    assert np.all(err <= bound), f"{what}: max abs {err.max():.3e} at {worst}"


def oracle_weight(W, codebook=Q):
    ref = occ.quantize(W.float().numpy(), codebook)
    Wd = occ.dequantize(ref["packed"], ref["e"], ref["c2"], ref["mean"], codebook)
    return occ.bf16_bits_to_f32(Wd).reshape(W.shape).astype(np.float64)


def oracle_weight_f16(W, codebook=Q):
    """The weight as the fp16 compute dtype expands it."""
    ref = occ.quantize(W.float().numpy(), codebook)
    bits = occ.dequantize_f16(ref["packed"], ref["e"], ref["c2"], ref["mean"], codebook)
    return bits.view(np.float16).reshape(W.shape).astype(np.float64)


class Runner:
    """Quantizes W on the GPU and runs the layer through the C ABI."""

    def __init__(self, q, case, codebook=None):
        self.q, self.c = q, case
        N, K = case["W"].shape
        self.w = q.NF4Weight(N, K, codebook=codebook)
        ws = torch.empty(q.qlora_quantize_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")
        q.qlora_quantize_nf4_dq(case["W"].cuda(), self.w, ws)
        self.X = case["X"].cuda()
        self.A = case["A"].cuda()
        self.B = case["B"].cuda()
        self.dY = case["dY"].cuda()
        self.M = case["X"].shape[0]
        self.ws = torch.empty(q.qlora_linear_workspace_bytes(self.M, N, K, case["r"]), dtype=torch.uint8,
                              device="cuda")

    def fwd(self, ydt=torch.float32, save_h=False):
        N = self.w.rows
        Y = torch.empty(self.M, N, dtype=ydt, device="cuda")
        H = torch.empty(self.M, self.c["r"], dtype=torch.float32, device="cuda") if save_h else None
        self.q.qlora_linear_fwd(self.w, self.X, self.M, self.A, self.B, self.c["r"], self.c["scale"], Y, H, self.ws)
        self.q.qlora_check_device_error()
        return Y, H

    def bwd(self, dxdt=torch.float32, H=None, want_dx=True):
        N, K, r = self.w.rows, self.w.cols, self.c["r"]
        dX = torch.empty(self.M, K, dtype=dxdt, device="cuda") if want_dx else None
        dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
        dB = torch.empty(N, r, dtype=torch.float32, device="cuda")
        self.q.qlora_linear_bwd(self.w, self.X, self.dY, self.M, self.A, self.B, r, self.c["scale"], H, dX, dA, dB,
                                self.ws)
        self.q.qlora_check_device_error()
        return dX, dA, dB


def np64(t):
    return t.float().cpu().numpy().astype(np.float64)


def full_check(q, case, ydt=torch.float32, codebook=None):
    run = Runner(q, case, codebook)
    Wd = oracle_weight(case["W"], Q if codebook is None else np.asarray(codebook, np.float32))
    X, A, B, dY = (np64(case[k]) for k in ("X", "A", "B", "dY"))
    s = case["scale"]
    Y, _ = run.fwd(ydt)
    assert_close(np64(Y), olin.forward(X, Wd, A, B, s), bf16_out=ydt == torch.bfloat16, what="Y")
    dX, dA, dB = run.bwd(ydt)
    rdX, rdA, rdB = olin.backward(X, Wd, A, B, s, dY)
    assert_close(np64(dX), rdX, bf16_out=ydt == torch.bfloat16, what="dX")
    assert_close(np64(dA), rdA, what="dA")
    assert_close(np64(dB), rdB, what="dB")
    return run


def test_tiny_config(q):
    full_check(q, synthetic.tiny_linear(seed=0))


def test_tiny_config_bf16_outputs(q):
    full_check(q, synthetic.tiny_linear(seed=0), ydt=torch.bfloat16)


@pytest.mark.parametrize("M,N,K,r", [
    (300, 320, 448, 16),     # ragged tails in every dimension, several tiles
    (129, 512, 256, 64),     # one token past a tile
    (64, 264, 576, 8),       # N not a multiple of 64
    (256, 256, 1024, 128),   # largest rank
    (1, 512, 512, 64),       # a single token
])
def test_ragged_shapes(q, M, N, K, r):
    full_check(q, synthetic.linear_case(M, N, K, r, alpha=16.0, seed=M + N + K + r))


@pytest.mark.parametrize("M,N,K,r", [
    (300, 320, 448, 16),     # CTA pairs, ragged in every dimension
    (600, 264, 576, 64),     # two pair tiles of tokens, N not a multiple of the 256-wide pair tile
    (513, 512, 256, 128),    # one token into the second pair tile, largest rank
])
def test_ragged_shapes_bf16_outputs(q, M, N, K, r):
    """bf16 Y and dX through the CTA-pair kernels' TMA-store epilogue (the
    tensor map clips the ragged edges)."""
    full_check(q, synthetic.linear_case(M, N, K, r, alpha=16.0, seed=2 * M + N + K + r), ydt=torch.bfloat16)


@pytest.mark.parametrize("M", [17, 200, 256])
def test_single_cta_fused_bf16_outputs(q, M):
    """17..256 tokens: the single-CTA fused forward and input-gradient GEMMs
    with bf16 outputs (one 256-token tile)."""
    full_check(q, synthetic.linear_case(M, 384, 512, 64, alpha=16.0, seed=300 + M), ydt=torch.bfloat16)


@pytest.mark.parametrize("M,N,K", [(17, 1024, 4096), (200, 1024, 4096), (256, 4096, 4096), (100, 512, 8192)])
@pytest.mark.parametrize("ydt", [torch.float32, torch.bfloat16])
def test_single_cta_split_contraction(q, M, N, K, ydt):
    """17..256 tokens with few output tiles: the single-CTA fused forward and
    input gradient split the contraction over idle SMs (fp32 planes summed in
    order by a second kernel)."""
    full_check(q, synthetic.linear_case(M, N, K, 64, alpha=16.0, seed=500 + M + N), ydt=ydt)


@pytest.mark.parametrize("M", [16, 200, 512])
def test_int4_codebook(q, M):
    """The Int4 table through the same kernels: the decode forward (16
    tokens), the single-CTA fused GEMMs (200) and the CTA-pair GEMMs (512)."""
    case = synthetic.linear_case(M, 384, 320, 16, alpha=16.0, seed=70 + M)
    table = q.qlora_build_int4_codebook()
    assert np.array_equal(np.array(table, np.float32).view(np.uint32), ocb.int4_codebook().view(np.uint32))
    full_check(q, case, codebook=table)


@pytest.mark.parametrize("M", [16, 200, 512])
def test_fp4_codebook(q, M):
    """The FP4 (E2M1) table through the decode (16 tokens), single-CTA (200)
    and CTA-pair (512) kernels, with bf16 outputs."""
    case = synthetic.linear_case(M, 384, 320, 16, alpha=16.0, seed=80 + M)
    full_check(q, case, ydt=torch.bfloat16, codebook=q.qlora_build_fp4_codebook())


def test_saved_h_equals_recomputed_h(q):
    case = synthetic.linear_case(200, 384, 512, 64, alpha=16.0, seed=5)
    run = Runner(q, case)
    _, H = run.fwd(save_h=True)
    X, A = np64(case["X"]), np64(case["A"])
    np.testing.assert_allclose(np64(H), case["scale"] * X @ A.T, rtol=1e-5, atol=1e-5)
    a = run.bwd(H=None)
    b = run.bwd(H=H)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_without_input_gradient(q):
    case = synthetic.linear_case(128, 256, 256, 16, alpha=32.0, seed=6)
    run = Runner(q, case)
    dX0, dA0, dB0 = run.bwd()
    dX, dA, dB = run.bwd(want_dx=False)
    assert dX is None and torch.equal(dA, dA0) and torch.equal(dB, dB0)


def test_zero_adapter_and_zero_scale(q):
    case = synthetic.linear_case(130, 256, 320, 16, alpha=16.0, seed=8)
    case["B"] = torch.zeros_like(case["B"])
    run = Runner(q, case)
    Wd = oracle_weight(case["W"])
    Y, _ = run.fwd()
    assert_close(np64(Y), np64(case["X"]) @ Wd.T, what="Y with B = 0")
    dX, dA, dB = run.bwd()
    assert torch.count_nonzero(dA).item() == 0, "G = 0 gives dA = 0 exactly"
    case = synthetic.linear_case(130, 256, 320, 16, alpha=0.0, seed=9)
    run = Runner(q, case)
    dX, dA, dB = run.bwd()
    assert torch.count_nonzero(dA).item() == 0 and torch.count_nonzero(dB).item() == 0


def test_zero_tokens(q):
    case = synthetic.linear_case(4, 128, 128, 8, alpha=16.0, seed=10)
    run = Runner(q, case)
    run.M = 0
    dX, dA, dB = run.bwd(want_dx=False)
    assert torch.count_nonzero(dA).item() == 0 and torch.count_nonzero(dB).item() == 0


def test_deterministic(q):
    case = synthetic.linear_case(512, 512, 1024, 64, alpha=16.0, seed=12)
    run = Runner(q, case)
    y1, _ = run.fwd()
    y2, _ = run.fwd()
    assert torch.equal(y1, y2)
    g1, g2 = run.bwd(), run.bwd()
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


@pytest.mark.parametrize("ydt", [torch.bfloat16, torch.float32])
def test_llama7b_shapes_sampled(q, ydt):
    """7B-shaped linears at 4096 tokens: Y and dX on sampled rows, dA and dB in
    full (they contract over every token).  With bf16 outputs and the saved H
    this is exactly the call sequence the benchmark times (the CTA-pair
    kernels with the TMA-store epilogue)."""
    rng = np.random.default_rng(0)
    bf = ydt == torch.bfloat16
    for i, (name, N, K) in enumerate([("q", 4096, 4096), ("gate", 11008, 4096), ("down", 4096, 11008)]):
        case = synthetic.linear_case(4096, N, K, 64, alpha=16.0, seed=100 + i, device="cpu")
        run = Runner(q, case)
        Wd = oracle_weight(case["W"])
        X, A, B, dY = (np64(case[k]) for k in ("X", "A", "B", "dY"))
        s = case["scale"]
        rows = np.sort(rng.choice(4096, 48, replace=False))
        Y, H = run.fwd(ydt, save_h=bf)
        assert_close(np64(Y)[rows], olin.forward_rows(X, Wd, A, B, s, rows), bf16_out=bf, what=f"{name} Y")
        dX, dA, dB = run.bwd(ydt, H=H)
        assert_close(np64(dX)[rows], olin.backward_dx_rows(Wd, A, B, s, dY, rows), bf16_out=bf, what=f"{name} dX")
        rdA, rdB = olin.backward_weight_grads(X, A, B, s, dY)
        assert_close(np64(dA), rdA, what=f"{name} dA")
        assert_close(np64(dB), rdB, what=f"{name} dB")


def test_llama65b_shapes_sampled(q):
    """65B-shaped linears at 2048 tokens with bf16 Y and dX and the saved H, as
    the 80-layer stack benchmark calls them: Y and dX on sampled rows, dA and
    dB in full."""
    rng = np.random.default_rng(1)
    for i, (name, N, K) in enumerate([("q", 8192, 8192), ("gate", 22016, 8192), ("down", 8192, 22016)]):
        case = synthetic.linear_case(2048, N, K, 64, alpha=16.0, seed=500 + i, device="cpu")
        run = Runner(q, case)
        Wd = oracle_weight(case["W"])
        X, A, B, dY = (np64(case[k]) for k in ("X", "A", "B", "dY"))
        s = case["scale"]
        rows = np.sort(rng.choice(2048, 32, replace=False))
        Y, H = run.fwd(torch.bfloat16, save_h=True)
        assert_close(np64(Y)[rows], olin.forward_rows(X, Wd, A, B, s, rows), bf16_out=True, what=f"{name} Y")
        dX, dA, dB = run.bwd(torch.bfloat16, H=H)
        assert_close(np64(dX)[rows], olin.backward_dx_rows(Wd, A, B, s, dY, rows), bf16_out=True, what=f"{name} dX")
        rdA, rdB = olin.backward_weight_grads(X, A, B, s, dY)
        assert_close(np64(dA), rdA, what=f"{name} dA")
        assert_close(np64(dB), rdB, what=f"{name} dB")


def test_argument_errors(q):
    case = synthetic.linear_case(16, 128, 128, 8, alpha=16.0, seed=13)
    run = Runner(q, case)
    Y = torch.empty(16, 128, dtype=torch.float32, device="cuda")
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(q.QLoraError) as e:
        q.qlora_linear_fwd(run.w, run.X, 16, run.A, run.B, 8, 2.0, Y, None, small)
    assert e.value.status == 4
    with pytest.raises(q.QLoraError) as e:
        q.qlora_linear_fwd(run.w, run.X, 16, run.A, run.B, 12, 2.0, Y, None, run.ws)
    assert e.value.status == 2


@pytest.mark.parametrize("M,N,K,r,p", [
    (16, 384, 320, 16, 0.1),      # decode forward
    (200, 384, 512, 64, 0.05),    # single-CTA fused GEMMs
    (600, 264, 576, 64, 0.5),     # CTA pairs, ragged
    (4096, 4096, 4096, 64, 0.05), # LLaMA-7B attention shape, the blog's p
])
def test_lora_dropout(q, M, N, K, r, p):
    """LoRA dropout on the adapter input (the blog's LoraConfig snippet,
    lora_dropout): Y, dX (bf16) and dA, dB against the oracle on the same
    mask; the frozen path sees the undropped input."""
    case = synthetic.linear_case(M, N, K, r, alpha=16.0, seed=3000 + M)
    keep, packed = synthetic.dropout_mask(M, K, p, seed=3100 + M, device="cuda")
    run = Runner(q, case)
    run.ws = torch.empty(q.qlora_linear_workspace_bytes(M, N, K, r, dropout=(packed, p)), dtype=torch.uint8,
                         device="cuda")
    s = case["scale"]
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    H = torch.empty(M, r, dtype=torch.float32, device="cuda")
    q.qlora_linear_fwd(run.w, run.X, M, run.A, run.B, r, s, Y, H, run.ws, dropout=(packed, p))
    dX = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
    dB = torch.empty(N, r, dtype=torch.float32, device="cuda")
    q.qlora_linear_bwd(run.w, run.X, run.dY, M, run.A, run.B, r, s, H, dX, dA, dB, run.ws, dropout=(packed, p))
    q.qlora_check_device_error()
    Wd = oracle_weight(case["W"])
    X, A, B, dY = (np64(case[k]) for k in ("X", "A", "B", "dY"))
    keep = keep.numpy()
    Xd = olin.dropout_input(case["X"].float().numpy(), keep, p)
    rows = np.arange(M) if M <= 600 else np.sort(np.random.default_rng(7).choice(M, 48, replace=False))
    rY = olin.forward_dropout(X[rows], Wd, A, B, s, Xd[rows])
    assert_close(np64(Y)[rows], rY, bf16_out=True, what="Y")
    np.testing.assert_allclose(np64(H), s * Xd @ A.T, rtol=1e-5, atol=1e-5)
    rdX, rdA, rdB = olin.backward_dropout(X, Wd, A, B, s, dY, Xd, keep, p) if M <= 600 else (None, None, None)
    if rdX is None:
        G = dY @ B
        rdX = (dY[rows] @ Wd) + s * (G[rows] @ A) * (keep[rows] * np.float64(olin.dropout_scale(p)))
        rdA, rdB = s * (G.T @ Xd), s * (dY.T @ (Xd @ A.T))
        assert_close(np64(dX)[rows], rdX, bf16_out=True, what="dX")
    else:
        assert_close(np64(dX), rdX, bf16_out=True, what="dX")
    assert_close(np64(dA), rdA, what="dA")
    assert_close(np64(dB), rdB, what="dB")



@pytest.mark.parametrize("M", [16, 200, 600])
@pytest.mark.parametrize("odt", [torch.float16, torch.float32])
def test_fp16_compute_dtype(q, M, odt):
    """The fp16 compute dtype (the blog's BitsAndBytesConfig snippet,
    bnb_4bit_compute_dtype=torch.float16): fp16 X, A, B, dY, the weight
    expanded to fp16, fp16 or fp32 outputs; through the decode (16 tokens),
    single-CTA (200) and CTA-pair (600) kernels."""
    case = synthetic.linear_case(M, 384, 512, 64, alpha=16.0, seed=4000 + M, act_dtype=torch.float16)
    run = Runner(q, case)
    Wd = oracle_weight_f16(case["W"])
    X, A, B, dY = (np64(case[k]) for k in ("X", "A", "B", "dY"))
    s = case["scale"]
    f16 = odt == torch.float16
    Y, H = run.fwd(odt, save_h=True)
    assert_close(np64(Y), olin.forward(X, Wd, A, B, s), f16_out=f16, what="Y")
    dX, dA, dB = run.bwd(odt, H=H)
    rdX, rdA, rdB = olin.backward(X, Wd, A, B, s, dY)
    assert_close(np64(dX), rdX, f16_out=f16, what="dX")
    assert_close(np64(dA), rdA, what="dA")
    assert_close(np64(dB), rdB, what="dB")


def test_fp16_compute_dtype_llama7b_gate(q):
    """fp16 compute dtype at the LLaMA-7B gate shape (11008 x 4096), 4096 tokens:
    Y and dX on sampled rows, dA and dB in full."""
    case = synthetic.linear_case(4096, 11008, 4096, 64, alpha=16.0, seed=4100, act_dtype=torch.float16)
    run = Runner(q, case)
    Wd = oracle_weight_f16(case["W"])
    X, A, B, dY = (np64(case[k]) for k in ("X", "A", "B", "dY"))
    s = case["scale"]
    rows = np.sort(np.random.default_rng(11).choice(4096, 48, replace=False))
    Y, H = run.fwd(torch.float16, save_h=True)
    assert_close(np64(Y)[rows], olin.forward_rows(X, Wd, A, B, s, rows), f16_out=True, what="Y")
    dX, dA, dB = run.bwd(torch.float16, H=H)
    assert_close(np64(dX)[rows], olin.backward_dx_rows(Wd, A, B, s, dY, rows), f16_out=True, what="dX")
    rdA, rdB = olin.backward_weight_grads(X, A, B, s, dY)
    assert_close(np64(dA), rdA, what="dA")
    assert_close(np64(dB), rdB, what="dB")


def _whole_or_split(q, run, ydt, dropout, split, side=None, divide_bwd=False):
    """Forward then backward, either as single calls or with the adapter
    products split off (optionally on a side stream, ordered by events);
    divide_bwd: the rest of the backward as two calls, dA and dB on the side
    stream and dX on the main one."""
    M, N, K, r, s = run.M, run.w.rows, run.w.cols, run.c["r"], run.c["scale"]
    ws = torch.zeros(q.qlora_linear_workspace_bytes(M, N, K, r, dropout=dropout), dtype=torch.uint8, device="cuda")
    Y = torch.empty(M, N, dtype=ydt, device="cuda")
    H = torch.empty(M, r, dtype=torch.float32, device="cuda")
    dX = torch.empty(M, K, dtype=ydt, device="cuda")
    dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
    dB = torch.empty(N, r, dtype=torch.float32, device="cuda")
    main = torch.cuda.current_stream()
    args_f = (run.w, run.X, M, run.A, run.B, r, s)
    args_b = (run.w, run.X, run.dY, M, run.A, run.B, r, s, H)
    if not split:
        q.qlora_linear_fwd(*args_f, Y, H, ws, dropout=dropout)
        q.qlora_linear_bwd(*args_b, dX, dA, dB, ws, dropout=dropout)
    else:
        for phase in ("fwd", "bwd"):
            st = side if side is not None else main
            st.wait_stream(main)
            with torch.cuda.stream(st):
                if phase == "fwd":
                    q.qlora_linear_adapter_fwd(*args_f, H, ws, stream=st, dropout=dropout)
                else:
                    q.qlora_linear_adapter_bwd(*args_b, ws, stream=st, dropout=dropout)
            main.wait_stream(st)
            if phase == "fwd":
                q.qlora_linear_fwd(*args_f, Y, H, ws, dropout=dropout, adapter_ready=True)
            elif divide_bwd:
                q.qlora_linear_bwd(*args_b, dX, None, None, ws, dropout=dropout, adapter_ready=True)
                with torch.cuda.stream(st):
                    q.qlora_linear_bwd(*args_b, None, dA, dB, ws, stream=st, dropout=dropout, adapter_ready=True)
                main.wait_stream(st)
            else:
                q.qlora_linear_bwd(*args_b, dX, dA, dB, ws, dropout=dropout, adapter_ready=True)
    q.qlora_check_device_error()
    return Y, H, dX, dA, dB


@pytest.mark.parametrize("M,p", [(512, None), (600, 0.1), (200, None), (16, None), (16, 0.1), (4096, None)])
@pytest.mark.parametrize("ydt", [torch.bfloat16, torch.float32])
def test_adapter_split_equals_whole_call(q, M, p, ydt):
    """The adapter products run on their own first (qlora_linear_adapter_fwd /
    _bwd, on a side stream for the CTA-pair sizes), then the rest of each
    call with adapter_ready: the same bits as the undivided calls, for the
    CTA-pair, single-CTA and decode paths, with and without LoRA dropout."""
    N, K, r = (4096, 4096, 64) if M == 4096 else (384, 512, 64)
    run = Runner(q, synthetic.linear_case(M, N, K, r, alpha=16.0, seed=4000 + M))
    dropout = None
    if p is not None:
        _, packed = synthetic.dropout_mask(M, K, p, seed=4100 + M, device="cuda")
        dropout = (packed, p)
    side = torch.cuda.Stream() if M > 256 else None
    whole = _whole_or_split(q, run, ydt, dropout, split=False)
    split = _whole_or_split(q, run, ydt, dropout, split=True, side=side)
    for name, a, b in zip(("Y", "H", "dX", "dA", "dB"), whole, split):
        assert torch.equal(a, b), name
    divided = _whole_or_split(q, run, ydt, dropout, split=True, side=side or torch.cuda.Stream(), divide_bwd=True)
    for name, a, b in zip(("Y", "H", "dX", "dA", "dB"), whole, divided):
        assert torch.equal(a, b), "divided backward: " + name
