"""qlora_quantize_nf4_dq_noalloc: the quantizer with the library's fixed scratch
array instead of a caller workspace.

It must write the same bytes as qlora_quantize_nf4_dq (whose parity with the
oracle is tested in test_gpu_codec.py) on consecutive calls that reuse the
scratch array, and refuse weights larger than the array before touching the
GPU.  This file is named to run last, so that it also passes after every
other test has used the library on the same device.
"""

import ctypes
import os

import numpy as np
import pytest
import torch

import synthetic

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "..", "bit_nf4_quantized_16_b200", "libqlora_b200.so")
MAX_BLOCKS = 1 << 20


class Weight(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("packed", ctypes.c_void_p),
                ("code2", ctypes.c_void_p), ("c2", ctypes.c_void_p), ("mean", ctypes.c_void_p),
                ("codebook", ctypes.c_float * 16)]


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        pytest.skip("library not built")
    lib = ctypes.CDLL(LIB)
    lib.qlora_quantize_nf4_dq_noalloc.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(Weight),
                                                  ctypes.c_void_p]
    lib.qlora_quantize_nf4_dq_noalloc.restype = ctypes.c_int
    return lib


def _codebook(lib):
    out = (ctypes.c_float * 16)()
    lib.qlora_build_nf4_codebook.argtypes = [ctypes.c_double, ctypes.c_void_p]
    assert lib.qlora_build_nf4_codebook(0.0, ctypes.cast(out, ctypes.c_void_p)) == 0
    return list(out)


def test_header_limit_matches_binding():
    import bit_nf4_quantized_16_b200 as q
    assert q.QLORA_NOALLOC_MAX_BLOCKS == MAX_BLOCKS
    header = open(os.path.join(HERE, "..", "include", "qlora.h")).read()
    assert "#define QLORA_NOALLOC_MAX_BLOCKS (1 << 20)" in header


def test_oversize_and_bad_arguments_rejected_before_any_cuda_call(lib):
    fake = 1 << 12   # never dereferenced: every check below fails first
    q = _codebook(lib)
    f = lib.qlora_quantize_nf4_dq_noalloc
    at_limit = Weight(MAX_BLOCKS // 64, 64 * 64, fake, fake, fake, fake, (ctypes.c_float * 16)(*q))
    over = Weight(MAX_BLOCKS // 64 + 1, 64 * 64, fake, fake, fake, fake, (ctypes.c_float * 16)(*q))
    assert at_limit.rows * at_limit.cols // 64 == MAX_BLOCKS
    assert f(fake, 0, ctypes.byref(over), None) == 2          # QLORA_ERR_SHAPE: larger than the scratch
    assert f(None, 0, ctypes.byref(at_limit), None) == 1      # null W
    assert f(fake, 9, ctypes.byref(at_limit), None) == 1      # unknown dtype
    assert f(fake + 4, 0, ctypes.byref(at_limit), None) == 3  # misaligned W
    ragged = Weight(64, 100, fake, fake, fake, fake, (ctypes.c_float * 16)(*q))
    assert f(fake, 0, ctypes.byref(ragged), None) == 2        # cols % 64


def _quantize_both(q, W):
    rows, cols = W.shape
    a = q.NF4Weight(rows, cols, device="cuda")
    b = q.NF4Weight(rows, cols, device="cuda")
    for t in (a.packed, a.code2, b.packed, b.code2):
        t.fill_(0xAB)
    a.c2.fill_(-1.0)
    b.c2.fill_(-2.0)
    ws = torch.empty(q.qlora_quantize_workspace_bytes(rows, cols), dtype=torch.uint8, device="cuda")
    q.qlora_quantize_nf4_dq(W, a, ws)
    q.qlora_quantize_nf4_dq_noalloc(W, b)
    torch.cuda.synchronize()
    return a, b


def _assert_same(a, b):
    assert torch.equal(a.packed, b.packed), "packed codes"
    assert torch.equal(a.code2, b.code2), "E4M3 codes"
    assert torch.equal(a.c2.view(torch.int32), b.c2.view(torch.int32)), "group scales"
    assert a.mean[0].view(torch.int32).item() == b.mean[0].view(torch.int32).item(), "mean"


@pytest.mark.gpu
def test_consecutive_calls_match_the_workspace_entry_point():
    import bit_nf4_quantized_16_b200 as q
    assert torch.cuda.is_available()
    # a large bf16 weight, then a small ragged fp32 one (its groups and mean
    # must not see the first call's leftovers in the shared scratch), then the
    # weight at the size limit, then the first weight again
    W1 = synthetic.normal((4096, 11008), 0.02, seed=101).to(torch.bfloat16).cuda()
    W2 = synthetic.normal((257, 320), 1.0, seed=102).cuda()
    W3 = synthetic.normal((8192, 8192), 0.02, seed=103).to(torch.bfloat16).cuda()
    assert W3.numel() // 64 == MAX_BLOCKS
    first = None
    for W in (W1, W2, W3, W1):
        a, b = _quantize_both(q, W)
        _assert_same(a, b)
        if first is None:
            first = b
        elif W is W1:
            _assert_same(first, b)   # deterministic across calls that reuse the scratch


@pytest.mark.gpu
def test_oversize_weight_rejected_on_the_gpu_path():
    import bit_nf4_quantized_16_b200 as q
    rows, cols = MAX_BLOCKS // 64 + 1, 64 * 64
    w = q.NF4Weight(rows, cols, device="cuda")
    W = torch.zeros(rows, cols, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError, match="QLORA_ERR_SHAPE"):
        q.qlora_quantize_nf4_dq_noalloc(W, w)
