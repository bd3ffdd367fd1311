"""NF4 + double-quantization codec, oracle side (driver for nf4_ref.c).

TEST INFRASTRUCTURE (see the package docstring).

Layout of a quantized [rows, cols] tensor (cols % 64 == 0), shared by the
oracle and the CUDA library because it is the storage format itself:
  packed  uint8 [rows*cols/2]   element 2j in the low nibble of byte j,
                                element 2j+1 in the high nibble (row-major)
  e       uint8 [nblocks]       E4M3 code of (c1_b - mean) / c2_g per block
  c2      float32 [ngroups]     second-level scale per group of 256 blocks
  mean    float32               one per tensor
nblocks = rows*cols/64, blocks in row-major order; ngroups = ceil(nblocks/256).
"""

import ctypes
import os
import subprocess

import numpy as np

from . import exact

BLOCK = 64
GROUP = 256

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nf4_ref.c")
_LIB = os.path.join(_HERE, "_nf4_ref.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile nf4_ref.c with gcc (no contraction of multiply-adds)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
            "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", _LIB, "-lm",
        ])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        lib.oracle_bf16_rne.restype = ctypes.c_uint16
        lib.oracle_bf16_rne.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_quantize_blocks.argtypes = [P, ctypes.c_int64, P, P, P]
        lib.oracle_pack_nibbles.argtypes = [P, ctypes.c_int64, P]
        lib.oracle_unpack_nibbles.argtypes = [P, ctypes.c_int64, P]
        lib.oracle_dq_encode.argtypes = [P, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, P, P]
        lib.oracle_dequantize.argtypes = [P, P, P, ctypes.c_float, P, ctypes.c_int64,
                                          ctypes.c_int32, P]
        lib.oracle_dequantize_f32.argtypes = [P, P, P, ctypes.c_float, P, ctypes.c_int64,
                                              ctypes.c_int32, P]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---- scalar helpers -------------------------------------------------------

def bf16_rne(x: np.ndarray) -> np.ndarray:
    """binary32 -> bf16 bit patterns (uint16), round to nearest even."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    return np.array([lib.oracle_bf16_rne(float(v)) for v in x.ravel()],
                    dtype=np.uint16).reshape(x.shape)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def e4m3_value(code: int) -> float:
    return _load().oracle_e4m3_value(code)


def e4m3_encode(t: float) -> int:
    return _load().oracle_e4m3_encode(t)


# ---- codec ------------------------------------------------------------------

def quantize_first_level(W: np.ndarray, q: np.ndarray):
    """c1 (float32 [nblocks]) and codes (uint8 [numel]) of a finite tensor."""
    lib = _load()
    x = np.ascontiguousarray(W, dtype=np.float32).ravel()
    if x.size % BLOCK:
        raise ValueError("element count must be a multiple of 64")
    nblocks = x.size // BLOCK
    q = np.ascontiguousarray(q, dtype=np.float32)
    c1 = np.empty(nblocks, np.float32)
    codes = np.empty(x.size, np.uint8)
    lib.oracle_quantize_blocks(_ptr(x), nblocks, _ptr(q), _ptr(c1), _ptr(codes))
    return c1, codes


def pack(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.size // 2, np.uint8)
    _load().oracle_pack_nibbles(_ptr(codes), codes.size, _ptr(out))
    return out


def unpack(packed: np.ndarray) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    out = np.empty(packed.size * 2, np.uint8)
    _load().oracle_unpack_nibbles(_ptr(packed), out.size, _ptr(out))
    return out


def dq_encode(c1: np.ndarray, mean: np.float32, group: int = GROUP):
    lib = _load()
    c1 = np.ascontiguousarray(c1, dtype=np.float32)
    ngroups = -(-c1.size // group)
    c2 = np.empty(ngroups, np.float32)
    e = np.empty(c1.size, np.uint8)
    lib.oracle_dq_encode(_ptr(c1), c1.size, group, float(mean), _ptr(c2), _ptr(e))
    return c2, e


def quantize(W: np.ndarray, q: np.ndarray, group: int = GROUP) -> dict:
    """Full NF4 + double quantization of W (any shape, numel % 64 == 0)."""
    c1, codes = quantize_first_level(W, q)
    mean = exact.exact_mean_f32(c1)
    c2, e = dq_encode(c1, mean, group)
    return {"packed": pack(codes), "e": e, "c2": c2, "mean": np.float32(mean),
            "c1": c1, "codes": codes}


def dequantize(packed, e, c2, mean, q, group: int = GROUP) -> np.ndarray:
    """bf16 bit patterns (uint16 [numel]) of the dequantized tensor."""
    lib = _load()
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    e = np.ascontiguousarray(e, dtype=np.uint8)
    c2 = np.ascontiguousarray(c2, dtype=np.float32)
    q = np.ascontiguousarray(q, dtype=np.float32)
    nblocks = e.size
    if packed.size != nblocks * BLOCK // 2:
        raise ValueError("packed / e size mismatch")
    w = np.empty(nblocks * BLOCK, np.uint16)
    lib.oracle_dequantize(_ptr(packed), _ptr(e), _ptr(c2), float(mean), _ptr(q),
                          nblocks, group, _ptr(w))
    return w


def dequantize_f16(packed, e, c2, mean, q, group: int = GROUP) -> np.ndarray:
    """fp16 bit patterns (uint16 [numel]) of the tensor dequantized for the fp16
    compute dtype: RN32(q[code] * c1') (C loops) rounded to nearest-even
    binary16 (numpy's conversion)."""
    lib = _load()
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    e = np.ascontiguousarray(e, dtype=np.uint8)
    c2 = np.ascontiguousarray(c2, dtype=np.float32)
    q = np.ascontiguousarray(q, dtype=np.float32)
    nblocks = e.size
    if packed.size != nblocks * BLOCK // 2:
        raise ValueError("packed / e size mismatch")
    w = np.empty(nblocks * BLOCK, np.float32)
    lib.oracle_dequantize_f32(_ptr(packed), _ptr(e), _ptr(c2), float(mean), _ptr(q),
                              nblocks, group, _ptr(w))
    return w.astype(np.float16).view(np.uint16)


def storage_bits_per_param(numel: int, group: int = GROUP) -> float:
    """Bits per parameter of the stored format (packed codes + e + c2 + mean)."""
    nblocks = numel // BLOCK
    ngroups = -(-nblocks // group)
    total_bytes = numel // 2 + nblocks + 4 * ngroups + 4
    return 8.0 * total_bytes / numel
