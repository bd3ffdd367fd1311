"""The C-ABI library loads without a GPU, exports every symbol the header
declares, and its host-only logic (codebook, status strings, workspace sizes,
argument validation before any CUDA call) behaves as documented."""

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import codebook as ocb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "bit_nf4_quantized_16_b200", "libqlora_b200.so")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        import importlib.util
        spec = importlib.util.spec_from_file_location("qbuild", os.path.join(ROOT, "bit_nf4_quantized_16_b200", "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build()
    return ctypes.CDLL(LIB)


def declared_symbols():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"QLORA_API\s+[\w\s\*]+?\b(qlora_\w+)\s*\(", txt)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n


def test_bounds_checked_build_exports_every_symbol():
    """The QLORA_DEBUG build (libqlora_b200_debug.so) is the same ABI."""
    path = os.path.join(ROOT, "bit_nf4_quantized_16_b200", "libqlora_b200_debug.so")
    if not os.path.exists(path):
        import importlib.util
        spec = importlib.util.spec_from_file_location("qbuild", os.path.join(ROOT, "bit_nf4_quantized_16_b200", "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build(debug=True)
    dlib = ctypes.CDLL(path)
    for n in declared_symbols():
        assert hasattr(dlib, n), n


def test_ordinary_build_has_no_bounds_checks(lib):
    """qlora_debug_bounds answers -1 and the self-test is unsupported (no CUDA call)."""
    lib.qlora_debug_bounds.restype = ctypes.c_int
    lib.qlora_debug_bounds.argtypes = [ctypes.c_char_p, ctypes.c_size_t]
    buf = ctypes.create_string_buffer(16)
    assert lib.qlora_debug_bounds(buf, 16) == -1 and buf.value == b""
    assert lib.qlora_debug_bounds_selftest() == 6   # QLORA_ERR_UNSUPPORTED


def test_binding_lists_the_same_symbols():
    src = open(os.path.join(ROOT, "bit_nf4_quantized_16_b200", "__init__.py")).read()
    exports = re.search(r"EXPORTS = \((.*?)\)", src, re.S).group(1)
    assert sorted(re.findall(r'"(qlora_\w+)"', exports)) == declared_symbols()


def test_nf4_codebook_matches_oracle_bit_for_bit(lib):
    out = (ctypes.c_float * 16)()
    lib.qlora_build_nf4_codebook.argtypes = [ctypes.c_double, ctypes.c_void_p]
    assert lib.qlora_build_nf4_codebook(0.0, ctypes.cast(out, ctypes.c_void_p)) == 0
    got = np.array(list(out), np.float32)
    assert np.array_equal(got.view(np.uint32), ocb.nf4_codebook().view(np.uint32))
    for delta in (0.01, 0.05, 0.1):
        assert lib.qlora_build_nf4_codebook(delta, ctypes.cast(out, ctypes.c_void_p)) == 0
        ref = ocb.nfk_codebook_f64(4, delta).astype(np.float32)
        assert np.array_equal(np.array(list(out), np.float32).view(np.uint32), ref.view(np.uint32))
    assert lib.qlora_build_nf4_codebook(0.5, ctypes.cast(out, ctypes.c_void_p)) == 1
    assert lib.qlora_build_nf4_codebook(0.0, None) == 1


def test_int4_codebook_matches_oracle_bit_for_bit(lib):
    out = (ctypes.c_float * 16)()
    lib.qlora_build_int4_codebook.argtypes = [ctypes.c_void_p]
    assert lib.qlora_build_int4_codebook(ctypes.cast(out, ctypes.c_void_p)) == 0
    got = np.array(list(out), np.float32)
    assert np.array_equal(got.view(np.uint32), ocb.int4_codebook().view(np.uint32))
    assert lib.qlora_build_int4_codebook(None) == 1


@pytest.mark.parametrize("k", [2, 3, 4])
def test_nfk_codebook_matches_oracle_bit_for_bit(lib, k):
    out = (ctypes.c_float * 16)()
    lib.qlora_build_nfk_codebook.argtypes = [ctypes.c_int, ctypes.c_double, ctypes.c_void_p]
    assert lib.qlora_build_nfk_codebook(k, 0.0, ctypes.cast(out, ctypes.c_void_p)) == 0
    got = np.array(list(out), np.float32)
    assert np.array_equal(got.view(np.uint32), ocb.nfk_table(k).view(np.uint32))
    assert lib.qlora_build_nfk_codebook(5, 0.0, ctypes.cast(out, ctypes.c_void_p)) == 1
    assert lib.qlora_build_nfk_codebook(3, 0.5, ctypes.cast(out, ctypes.c_void_p)) == 1


def test_fp4_codebook_matches_oracle_bit_for_bit(lib):
    out = (ctypes.c_float * 16)()
    lib.qlora_build_fp4_codebook.argtypes = [ctypes.c_void_p]
    assert lib.qlora_build_fp4_codebook(ctypes.cast(out, ctypes.c_void_p)) == 0
    got = np.array(list(out), np.float32)
    assert np.array_equal(got.view(np.uint32), ocb.fp4_codebook().view(np.uint32))
    assert lib.qlora_build_fp4_codebook(None) == 1


def test_status_strings(lib):
    lib.qlora_status_string.restype = ctypes.c_char_p
    assert lib.qlora_status_string(0) == b"QLORA_OK"
    assert lib.qlora_status_string(7) == b"QLORA_ERR_TIMEOUT"
    assert lib.qlora_status_string(99) == b"QLORA_ERR_UNKNOWN"


def test_quantize_workspace_size(lib):
    lib.qlora_quantize_workspace_bytes.restype = ctypes.c_size_t
    lib.qlora_quantize_workspace_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64]
    n = lib.qlora_quantize_workspace_bytes(4096, 4096)
    assert n >= 4 * 4096 * 4096 // 64 and n % 16 == 0


class Weight(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("packed", ctypes.c_void_p),
                ("code2", ctypes.c_void_p), ("c2", ctypes.c_void_p), ("mean", ctypes.c_void_p),
                ("codebook", ctypes.c_float * 16)]


def test_validation_happens_before_any_cuda_call(lib):
    """Bad arguments are rejected on the host; these calls never reach CUDA."""
    q = ocb.nf4_codebook()
    fake = 0x10000   # aligned, never dereferenced
    w = Weight(64, 128, fake, fake, fake, fake, (ctypes.c_float * 16)(*q))
    f = lib.qlora_quantize_nf4_dq
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(Weight), ctypes.c_void_p, ctypes.c_size_t,
                  ctypes.c_void_p]
    assert f(None, 0, ctypes.byref(w), fake, 1 << 20, None) == 1            # null W
    assert f(fake, 7, ctypes.byref(w), fake, 1 << 20, None) == 1            # bad dtype
    bad = Weight(64, 100, fake, fake, fake, fake, (ctypes.c_float * 16)(*q))
    assert f(fake, 0, ctypes.byref(bad), fake, 1 << 20, None) == 2          # cols % 64
    assert f(fake + 4, 0, ctypes.byref(w), fake, 1 << 20, None) == 3        # misaligned W
    assert f(fake, 0, ctypes.byref(w), fake, 16, None) == 4                 # workspace too small
    unsorted = Weight(64, 128, fake, fake, fake, fake, (ctypes.c_float * 16)(*q[::-1]))
    assert f(fake, 0, ctypes.byref(unsorted), fake, 1 << 20, None) == 1     # codebook not ascending


def _no_gpu():
    # the fake pointers below are never dereferenced because every call fails
    # validation first; still, never hand them to a library that sees a GPU
    try:
        import torch
        return not torch.cuda.is_available()
    except Exception:
        return True


@pytest.mark.skipif(not _no_gpu(), reason="host-only validation test with placeholder pointers")
def test_validation_of_tables_dequantize_and_noalloc(lib):
    q = ocb.nf4_codebook()
    fake = 0x10000
    quant = lib.qlora_quantize_nf4_dq
    quant.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(Weight), ctypes.c_void_p, ctypes.c_size_t,
                      ctypes.c_void_p]
    two_zeros = q.copy()
    two_zeros[8] = 0.0
    two_zeros[7] = np.float32(-1e-30)
    two_zeros[6] = 0.0
    w = Weight(64, 128, fake, fake, fake, fake, (ctypes.c_float * 16)(*two_zeros))
    assert quant(fake, 0, ctypes.byref(w), fake, 1 << 20, None) == 1          # not strictly ascending
    close = q.copy()
    close[12] = np.nextafter(close[11], np.float32(2))                        # 11, 12 almost equal:
    close[13] = np.nextafter(close[12], np.float32(2))                        # two midpoints, one interval
    w = Weight(64, 128, fake, fake, fake, fake, (ctypes.c_float * 16)(*close))
    assert quant(fake, 0, ctypes.byref(w), fake, 1 << 20, None) == 6          # QLORA_ERR_UNSUPPORTED
    noz = np.linspace(-1, 1, 17)[np.arange(17) != 8].astype(np.float32)       # no zero at all
    w = Weight(64, 128, fake, fake, fake, fake, (ctypes.c_float * 16)(*noz))
    assert quant(fake, 0, ctypes.byref(w), fake, 1 << 20, None) == 1

    deq = lib.qlora_dequantize_nf4_dq
    deq.argtypes = [ctypes.POINTER(Weight), ctypes.c_void_p, ctypes.c_void_p]
    w = Weight(64, 128, fake, fake, fake, fake, (ctypes.c_float * 16)(*q))
    assert deq(None, fake, None) == 1
    assert deq(ctypes.byref(w), None, None) == 1
    assert deq(ctypes.byref(w), fake + 2, None) == 3
    w_mis = Weight(64, 128, fake + 8, fake, fake, fake, (ctypes.c_float * 16)(*q))
    assert deq(ctypes.byref(w_mis), fake, None) == 3

    na = lib.qlora_quantize_nf4_dq_noalloc
    na.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(Weight), ctypes.c_void_p]
    big = Weight(1 << 14, 1 << 13, fake, fake, fake, fake, (ctypes.c_float * 16)(*q))   # 2^21 blocks
    assert na(fake, 0, ctypes.byref(big), None) == 2
    assert na(fake, 3, ctypes.byref(w), None) == 1


@pytest.mark.skipif(not _no_gpu(), reason="host-only validation test with placeholder pointers")
def test_validation_of_the_linear_layer(lib):
    q = ocb.nf4_codebook()
    fake = 0x10000
    P, I64, I32, F, S, I = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t,
                            ctypes.c_int)
    W = ctypes.POINTER(Weight)
    fwd = lib.qlora_linear_fwd
    fwd.argtypes = [W, P, I64, P, P, I32, F, P, I, P, P, S, P]
    bwd = lib.qlora_linear_bwd
    bwd.argtypes = [W, P, P, I64, P, P, I32, F, P, P, I, P, P, P, S, P]
    w = Weight(256, 256, fake, fake, fake, fake, (ctypes.c_float * 16)(*q))
    ok = dict(X=fake, M=16, A=fake, B=fake, r=16, Y=fake, ydt=1, H=None, ws=fake)

    def f(**kw):
        a = dict(ok, **kw)
        return fwd(kw.get("w", ctypes.byref(w)), a["X"], a["M"], a["A"], a["B"], a["r"], 1.0, a["Y"], a["ydt"],
                   a["H"], a["ws"], 1 << 30, None)

    assert f(M=-1) == 1
    assert f(r=0) == 2 and f(r=4) == 2 and f(r=12) == 2 and f(r=136) == 2
    assert f(X=None) == 1 and f(A=None) == 1 and f(B=None) == 1 and f(ws=None) == 1 and f(Y=None) == 1
    assert f(X=fake + 2) == 3 and f(B=fake + 8) == 3 and f(Y=fake + 4) == 3 and f(H=fake + 4) == 3
    assert f(ydt=5) == 1
    odd = Weight(250, 256, fake, fake, fake, fake, (ctypes.c_float * 16)(*q))
    assert f(w=ctypes.byref(odd)) == 2                                   # rows % 8
    assert f(w=None) == 1

    def b(**kw):
        a = dict(dict(ok, dY=fake, dX=fake, dA=fake, dB=fake, dxdt=1), **kw)
        return bwd(ctypes.byref(w), a["X"], a["dY"], a["M"], a["A"], a["B"], a["r"], 1.0, a["H"], a["dX"], a["dxdt"],
                   a["dA"], a["dB"], a["ws"], 1 << 30, None)

    assert b(dY=None) == 1 and b(dA=None) == 1 and b(dB=None) == 1
    assert b(dxdt=9) == 1
    assert b(dY=fake + 2) == 3 and b(dX=fake + 4) == 3 and b(dA=fake + 8) == 3 and b(H=fake + 4) == 3
    assert b(r=200) == 2


class Opts(ctypes.Structure):
    _fields_ = [("dropout_mask", ctypes.c_void_p), ("dropout_p", ctypes.c_float), ("compute_dtype", ctypes.c_int),
                ("adapter_ready", ctypes.c_int32)]


def test_validation_of_the_split_adapter_step(lib):
    """qlora_linear_adapter_fwd / _bwd and the adapter_ready option reject bad
    arguments before any CUDA call; the adapter calls need no output buffers."""
    q = ocb.nf4_codebook()
    fake = 0x10000
    P, I64, I32, F, S, I = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t,
                            ctypes.c_int)
    W, O = ctypes.POINTER(Weight), ctypes.POINTER(Opts)
    afwd = lib.qlora_linear_adapter_fwd
    afwd.argtypes = [W, P, I64, P, P, I32, F, P, P, S, P, O]
    abwd = lib.qlora_linear_adapter_bwd
    abwd.argtypes = [W, P, P, I64, P, P, I32, F, P, P, S, P, O]
    fwd_ex = lib.qlora_linear_fwd_ex
    fwd_ex.argtypes = [W, P, I64, P, P, I32, F, P, I, P, P, S, P, O]
    w = Weight(256, 256, fake, fake, fake, fake, (ctypes.c_float * 16)(*q))
    good = Opts(None, 0.0, 0, 0)

    def af(X=fake, M=64, A=fake, r=16, H=None, ws=fake, opts=good):
        return afwd(ctypes.byref(w), X, M, A, fake, r, 1.0, H, ws, 1 << 30, None,
                    None if opts is None else ctypes.byref(opts))

    def ab(dY=fake, M=64, r=16, H=None, opts=good):
        return abwd(ctypes.byref(w), fake, dY, M, fake, fake, r, 1.0, H, fake, 1 << 30, None,
                    None if opts is None else ctypes.byref(opts))

    assert af(X=None) == 1 and af(A=None) == 1 and af(ws=None) == 1 and af(M=-1) == 1
    assert af(r=12) == 2
    assert af(X=fake + 2) == 3 and af(H=fake + 4) == 3
    assert af(opts=Opts(None, 0.0, 0, 2)) == 1                 # adapter_ready is 0 or 1
    assert af(opts=Opts(None, 0.0, 9, 0)) == 1                 # unknown compute dtype
    assert af(opts=Opts(fake + 4, 0.1, 0, 0)) == 3             # misaligned dropout mask
    assert af(opts=Opts(fake, 1.0, 0, 0)) == 1                 # p outside [0, 1)
    assert ab(dY=None) == 1 and ab(dY=fake + 2) == 3 and ab(H=fake + 4) == 3 and ab(r=136) == 2
    assert ab(opts=Opts(None, 0.0, 0, 3)) == 1
    bwd_ex = lib.qlora_linear_bwd_ex
    bwd_ex.argtypes = [W, P, P, I64, P, P, I32, F, P, P, I, P, P, P, S, P, O]
    ready = Opts(None, 0.0, 0, 1)

    def b(dX=fake, dA=fake, dB=fake, opts=ready):
        return bwd_ex(ctypes.byref(w), fake, fake, 64, fake, fake, 16, 1.0, None, dX, 1, dA, dB, fake, 1 << 30, None,
                      ctypes.byref(opts))

    assert b(dA=None) == 1 and b(dB=None) == 1                   # dA and dB come together
    assert b(dX=None, dA=None, dB=None) == 1                     # nothing to form
    assert b(dA=None, dB=None, opts=good) == 1                   # the undivided backward needs dA, dB
    assert b(dA=None, dB=None, dX=fake + 4) == 3
    bad = Opts(None, 0.0, 0, 2)
    assert fwd_ex(ctypes.byref(w), fake, 64, fake, fake, 16, 1.0, fake, 1, None, fake, 1 << 30, None,
                  ctypes.byref(bad)) == 1


def test_stall_hook_validation(lib):
    """The failure-detection test hook only arms the kernel families that have
    pipeline waits, with a limit in range; it makes no CUDA call."""
    f = lib.qlora_debug_inject_stall
    f.argtypes = [ctypes.c_int, ctypes.c_uint64]
    assert f(5, 1_000_000) == 1             # low-rank products: not a hook site
    assert f(0, 10) == 1                    # limit below 1 us
    assert f(3, 3_000_000_000) == 1         # limit above 2 s
    assert f(-1, 0) == 0                    # disarm
    assert f(0, 1_000_000) == 0 and f(-1, 0) == 0


@pytest.mark.skipif(not _no_gpu(), reason="host-only validation test with placeholder pointers")
def test_shape_overflow_is_rejected(lib):
    """rows * cols that would overflow 64-bit arithmetic is rejected before use."""
    q = ocb.nf4_codebook()
    fake = 0x10000
    na = lib.qlora_quantize_nf4_dq_noalloc
    na.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(Weight), ctypes.c_void_p]
    huge = Weight(1 << 40, 1 << 30, fake, fake, fake, fake, (ctypes.c_float * 16)(*q))
    assert na(fake, 0, ctypes.byref(huge), None) == 2
    f = lib.qlora_quantize_nf4_dq
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(Weight), ctypes.c_void_p, ctypes.c_size_t,
                  ctypes.c_void_p]
    assert f(fake, 0, ctypes.byref(huge), fake, 1 << 62, None) == 2
