"""Pins of the oracle's NF4 + double-quantization codec.

"QLoRA: Efficient Finetuning of Quantized LLMs", section "Method":
"4-bit NormalFloat Quantization" (absmax rescaling into [-1, 1], step (3)) and
"Double Quantization" (constants of blocksize-64 blocks are quantized again).
"""

from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import codebook, codec, exact
from tests.conftest import read_golden

FIG = {k: float(v) for k, v in read_golden("paper_figures.txt")}
Q = codebook.nf4_codebook()


def _nearest_exact(n, q):
    """Index of the codebook value nearest to n in exact rational arithmetic,
    ties to the lower index."""
    dist = [abs(Fraction(float(n)) - Fraction(float(v))) for v in q]
    return min(range(len(q)), key=lambda j: (dist[j], j))


# ---- scalar formats -----------------------------------------------------------

def test_bf16_rne_against_torch():
    rng = np.random.default_rng(5)
    x = np.concatenate([
        rng.standard_normal(4000).astype(np.float32),
        # exact ties: low 16 bits == 0x8000, both parities of bit 16
        (rng.integers(0x3F000000, 0x40800000, 500, dtype=np.uint32) & 0xFFFF0000 | 0x8000).view(np.float32),
    ])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(codec.bf16_rne(x), ref)


@pytest.mark.parametrize("code_hex,value", read_golden("e4m3_spec.txt"))
def test_e4m3_spec_table(code_hex, value):
    v = codec.e4m3_value(int(code_hex, 16))
    assert v == float(value) and np.signbit(v) == np.signbit(float(value))


def test_e4m3_decode_all_codes_against_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        if c in (0x7F, 0xFF):
            assert np.isnan(ref[c])
            continue
        assert codec.e4m3_value(c) == ref[c]


def test_e4m3_encode_against_torch_and_ties():
    rng = np.random.default_rng(6)
    t = np.concatenate([
        rng.uniform(-448, 448, 3000), rng.standard_normal(2000) * 0.05,
        rng.standard_normal(500) * 1e-3,
    ]).astype(np.float32)
    # exact midpoints between neighbouring finite values: ties to even
    vals = np.array(sorted({codec.e4m3_value(c) for c in range(0x7F)}))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    t = np.concatenate([t, mids, -mids])
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([codec.e4m3_encode(float(v)) for v in t], np.uint8)
    assert np.array_equal(got, ref)
    for m in mids:
        c = codec.e4m3_encode(float(m))
        assert (c & 1) == 0, "ties go to the even mantissa"


def test_e4m3_encode_saturates_and_keeps_sign_of_zero():
    assert codec.e4m3_encode(500.0) == 0x7E
    assert codec.e4m3_encode(-1e30) == 0xFE
    assert codec.e4m3_encode(463.9) == 0x7E
    assert codec.e4m3_encode(1e-9) == 0x00
    assert codec.e4m3_encode(-1e-9) == 0x80


# ---- first level ----------------------------------------------------------------

def test_nearest_code_on_and_around_every_midpoint():
    """Blocks with absmax 1 (so n == x exactly): values on, just below and
    just above each exact midpoint between neighbouring codebook values."""
    xs = []
    for j in range(15):
        mid = (float(Q[j]) + float(Q[j + 1])) / 2          # exact in double
        m32 = np.float32(mid)
        xs += [m32, np.nextafter(m32, np.float32(-2)), np.nextafter(m32, np.float32(2))]
    xs = np.array(xs, np.float32)
    pad = (-xs.size) % 63
    body = np.concatenate([xs, np.zeros(pad, np.float32)]).reshape(-1, 63)
    W = np.concatenate([np.ones((body.shape[0], 1), np.float32), body], axis=1)
    c1, codes = codec.quantize_first_level(W, Q)
    assert np.all(c1 == 1.0)
    codes = codes.reshape(W.shape)
    for i in range(W.shape[0]):
        for k in range(64):
            assert codes[i, k] == _nearest_exact(W[i, k], Q), (W[i, k], codes[i, k])


def test_nearest_code_random_blocks_brute_force():
    rng = np.random.default_rng(7)
    W = (rng.standard_normal((8, 64)) * 0.02).astype(np.float32)
    c1, codes = codec.quantize_first_level(W, Q)
    assert np.array_equal(c1, np.abs(W).max(axis=1))
    for b in range(8):
        r = np.float32(1.0) / c1[b]
        for k in range(64):
            n = np.float32(W[b, k] * r)
            assert codes[64 * b + k] == _nearest_exact(n, Q)


def test_zero_and_subnormal_blocks_take_the_zero_code():
    W = np.zeros((3, 64), np.float32)
    W[1, 5] = 1e-40          # subnormal absmax
    W[2, :] = -0.0
    c1, codes = codec.quantize_first_level(W, Q)
    assert np.all(codes == 7)
    assert c1[1] == np.float32(1e-40)


def test_int4_table_nearest_code_and_zero_blocks():
    """The same first level with the Int4 table: values on, just below and
    just above every midpoint of the table take the nearest value (ties to
    the lower index), a zero block takes the table's zero (index 8), and
    bf16(q_j * a) inputs come back exactly."""
    q4 = codebook.int4_codebook()
    xs = []
    for j in range(15):
        m32 = np.float32((float(q4[j]) + float(q4[j + 1])) / 2)
        xs += [m32, np.nextafter(m32, np.float32(-2)), np.nextafter(m32, np.float32(2))]
    xs = [x for x in xs if abs(x) <= 1.0]
    xs = np.array(xs, np.float32)
    pad = (-xs.size) % 63
    body = np.concatenate([xs, np.zeros(pad, np.float32)]).reshape(-1, 63)
    W = np.concatenate([np.ones((body.shape[0], 1), np.float32), body], axis=1)
    c1, codes = codec.quantize_first_level(W, q4)
    assert np.all(c1 == 1.0)
    codes = codes.reshape(W.shape)
    for i in range(W.shape[0]):
        for k in range(64):
            assert codes[i, k] == _nearest_exact(W[i, k], q4), (W[i, k], codes[i, k])
    assert not np.any(codes == 0), "-8/7 is never the nearest value"
    _, zc = codec.quantize_first_level(np.zeros((2, 64), np.float32), q4)
    assert np.all(zc == 8)
    rng = np.random.default_rng(19)
    a = np.float32(0.0625)
    idx = rng.integers(1, 16, (16, 256)).astype(np.uint8)
    idx[:, ::64] = rng.choice([1, 15], (16, 4))
    Wr = codec.bf16_bits_to_f32(codec.bf16_rne((q4[idx] * a).astype(np.float32)))
    d = codec.quantize(Wr, q4)
    assert np.array_equal(d["codes"].reshape(idx.shape), idx)
    w = codec.dequantize(d["packed"], d["e"], d["c2"], d["mean"], q4)
    assert np.array_equal(codec.bf16_bits_to_f32(w), Wr.ravel())


def test_first_level_error_bound():
    """|x - q[code] c1| <= c1 * (largest half-gap of the codebook) + rounding."""
    rng = np.random.default_rng(8)
    W = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    c1, codes = codec.quantize_first_level(W, Q)
    half_gap = float(np.max(np.diff(Q.astype(np.float64)))) / 2
    approx = Q[codes].astype(np.float64).reshape(-1, 64) * c1[:, None]
    err = np.abs(approx - W.reshape(-1, 64))
    assert np.all(err <= c1[:, None] * (half_gap + 2.0 ** -22))


def test_pack_unpack_nibble_order():
    codes = np.array([1, 2, 15, 0, 7, 8], np.uint8)
    packed = codec.pack(codes)
    assert packed.tolist() == [0x21, 0x0F, 0x87]
    assert np.array_equal(codec.unpack(packed), codes)


# ---- double quantization and dequantization ---------------------------------------

def test_exact_round_trip_of_codebook_times_absmax():
    """W = bf16(q_j * a) with every block holding +-a: every c1 is a, the mean
    is a, c1 - mean = 0, c2 = 0, e = 0, and the dequantized tensor equals W."""
    rng = np.random.default_rng(9)
    a = np.float32(0.046875)                          # representable in bf16
    codes = rng.integers(0, 16, (32, 256)).astype(np.uint8)
    codes[:, ::64] = rng.choice([0, 15], (32, 4))     # +-1 in every block
    W = codec.bf16_bits_to_f32(codec.bf16_rne((Q[codes] * a).astype(np.float32)))
    d = codec.quantize(W, Q)
    assert np.array_equal(d["codes"].reshape(codes.shape), codes)
    assert d["mean"] == a and np.all(d["c2"] == 0) and np.all(d["e"] == 0)
    w = codec.dequantize(d["packed"], d["e"], d["c2"], d["mean"], Q)
    assert np.array_equal(codec.bf16_bits_to_f32(w), W.ravel())


def test_double_quantization_error_bound_and_groups():
    """E4M3 keeps 3 mantissa bits: |c1' - c1| <= amax_g * 2^-4 (+ rounding),
    groups are 256 consecutive blocks and the last one may be short."""
    rng = np.random.default_rng(10)
    W = (rng.standard_normal((1000, 64)) * 0.02).astype(np.float32)   # 1000 blocks
    d = codec.quantize(W, Q)
    assert d["c2"].size == 4
    mean = d["mean"]
    assert mean == exact.exact_mean_f32(d["c1"])
    ev = np.array([codec.e4m3_value(int(c)) for c in d["e"]])
    c1p = ev * np.repeat(d["c2"].astype(np.float64), 256)[:1000] + float(mean)
    for g in range(4):
        sl = slice(256 * g, min(256 * g + 256, 1000))
        amax = float(np.max(np.abs(d["c1"][sl].astype(np.float64) - float(mean))))
        assert d["c2"][g] == np.float32(amax / 448.0)
        bound = amax * 2.0 ** -4 + 2.0 ** -22 * (np.abs(d["c1"][sl]) + amax)
        assert np.all(np.abs(c1p[sl] - d["c1"][sl]) <= bound)


def test_dequantize_reproduces_definition_elementwise():
    """Spot check of the dequantizer against the definition, evaluated with
    exact rationals: c1' = RN32(e*c2 + mean), w = bf16(RN32(q*c1'))."""
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((4, 128)) * 0.02).astype(np.float32)
    d = codec.quantize(W, Q)
    w = codec.dequantize(d["packed"], d["e"], d["c2"], d["mean"], Q)
    for b in range(8):
        ev = Fraction(codec.e4m3_value(int(d["e"][b])))
        c1p = exact.rn32(ev * Fraction(float(d["c2"][b // 256])) + Fraction(float(d["mean"])))
        for k in range(0, 64, 7):
            code = int(d["codes"][64 * b + k])
            v = exact.rn32(Fraction(float(Q[code])) * Fraction(float(c1p)))
            ref = torch.tensor([float(v)], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item() & 0xFFFF
            assert int(w[64 * b + k]) == ref


def test_storage_bits_per_parameter_match_the_page():
    numel = 4096 * 4096
    bits = codec.storage_bits_per_param(numel)
    # 4-bit codes + one 8-bit code per 64 + one fp32 per 256*64 + the fp32 mean
    assert bits == pytest.approx(4 + 8 / 64 + 32 / (64 * 256) + 32 / numel, rel=1e-12)
    assert bits == pytest.approx(4.127, abs=5e-4)
    without_dq = FIG["k_bits"] + FIG["constant_bits"] / FIG["blocksize"]
    assert FIG["constant_bits"] / FIG["blocksize"] == FIG["constant_overhead_bits"]
    saving = without_dq - bits
    assert saving == pytest.approx(FIG["dq_saving_bits"], abs=0.005)
    assert 65e9 * saving / 8 / 1e9 == pytest.approx(FIG["dq_saving_65b_gb"], abs=0.1)



def test_fp16_dequantization_shares_the_products_of_the_bf16_one():
    """The fp16 compute dtype rounds the same binary32 products RN32(q * c1')
    to binary16: rounding those products to bf16 instead must give exactly the
    bf16 dequantizer's bits, and every fp16 value must be the nearest binary16
    of its product (checked against torch's conversion)."""
    import torch
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    q = codebook.nf4_codebook()
    ref = codec.quantize(W, q)
    h = codec.dequantize_f16(ref["packed"], ref["e"], ref["c2"], ref["mean"], q)
    lib = codec._load()
    prods = np.empty(W.size, np.float32)
    lib.oracle_dequantize_f32(codec._ptr(ref["packed"]), codec._ptr(ref["e"]), codec._ptr(ref["c2"]),
                              float(ref["mean"]), codec._ptr(q), ref["e"].size, 256, codec._ptr(prods))
    assert np.array_equal(codec.bf16_rne(prods),
                          codec.dequantize(ref["packed"], ref["e"], ref["c2"], ref["mean"], q))
    want = torch.from_numpy(prods).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(h, want)
