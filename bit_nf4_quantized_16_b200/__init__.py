"""Python binding of libqlora_b200.so (the C ABI declared in include/qlora.h).

Argument marshalling only: every function forwards to the C entry point of
the same name, passing torch device pointers and the current CUDA stream.
PyTorch provides device memory and streams; all arithmetic of the path runs
in the library's sm_100a kernels.  If the shared library is missing the
import fails loudly -- there is no fallback implementation.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# QLORA_B200_BUILD=debug selects the bounds-checked build (libqlora_b200_debug.so)
LIB_PATH = os.path.join(_HERE, "libqlora_b200_debug.so" if os.environ.get("QLORA_B200_BUILD") == "debug"
                        else "libqlora_b200.so")

QLORA_BLOCK = 64
QLORA_GROUP = 256
QLORA_NOALLOC_MAX_BLOCKS = 1 << 20   # largest rows*cols/64 of qlora_quantize_nf4_dq_noalloc
QLORA_BF16 = 0
QLORA_FP32 = 1
QLORA_FP16 = 2

STATUS = {
    0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_SHAPE", 3: "QLORA_ERR_ALIGNMENT",
    4: "QLORA_ERR_WORKSPACE", 5: "QLORA_ERR_CUDA", 6: "QLORA_ERR_UNSUPPORTED", 7: "QLORA_ERR_TIMEOUT",
}

# every symbol the header declares
EXPORTS = (
    "qlora_build_nf4_codebook", "qlora_build_nfk_codebook", "qlora_build_int4_codebook",
    "qlora_build_fp4_codebook",
    "qlora_quantize_workspace_bytes",
    "qlora_quantize_nf4_dq",
    "qlora_quantize_nf4_dq_noalloc",
    "qlora_dequantize_nf4_dq", "qlora_linear_workspace_bytes", "qlora_linear_fwd", "qlora_linear_bwd",
    "qlora_status_string", "qlora_check_device_error",
    "qlora_timing_enable", "qlora_timing_reset", "qlora_timing_read", "qlora_launch_count",
    "qlora_debug_inject_stall", "qlora_debug_bounds", "qlora_debug_bounds_selftest",
    "qlora_paged_alloc", "qlora_paged_free", "qlora_paged_prefetch", "qlora_adamw_step",
    "qlora_block_workspace_bytes", "qlora_block_fwd", "qlora_block_bwd",
    "qlora_linear_workspace_bytes_ex", "qlora_linear_fwd_ex", "qlora_linear_bwd_ex",
    "qlora_linear_adapter_fwd", "qlora_linear_adapter_bwd",
    "qlora_dequantize_nf4_dq_ex",
)

KERNEL_KINDS = ("quantize", "dq_encode", "dequantize", "fwd_fused", "bwd_fused", "lowrank", "wgrad",
                "elementwise", "optimizer", "block", "attention")


class QLoraError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}")
        self.status = status


class qlora_adamw_hparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("step", ctypes.c_int64)]


class qlora_nf4_weight(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
        ("packed", ctypes.c_void_p), ("code2", ctypes.c_void_p),
        ("c2", ctypes.c_void_p), ("mean", ctypes.c_void_p),
        ("codebook", ctypes.c_float * 16),
    ]


class qlora_linear_opts(ctypes.Structure):
    _fields_ = [("dropout_mask", ctypes.c_void_p), ("dropout_p", ctypes.c_float), ("compute_dtype", ctypes.c_int),
                ("adapter_ready", ctypes.c_int32)]


class qlora_block(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("seq", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("r", ctypes.c_int32), ("lora_scale", ctypes.c_float), ("rms_eps", ctypes.c_float),
                ("rope_base", ctypes.c_float), ("w", qlora_nf4_weight * 7), ("A", ctypes.c_void_p * 7),
                ("B", ctypes.c_void_p * 7), ("norm1", ctypes.c_void_p), ("norm2", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python bit_nf4_quantized_16_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I32, F, S = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    W = ctypes.POINTER(qlora_nf4_weight)
    sig = {
        "qlora_build_nf4_codebook": (ctypes.c_int, [ctypes.c_double, P]),
        "qlora_build_int4_codebook": (ctypes.c_int, [P]),
        "qlora_build_nfk_codebook": (ctypes.c_int, [ctypes.c_int, ctypes.c_double, P]),
        "qlora_build_fp4_codebook": (ctypes.c_int, [P]),
        "qlora_quantize_workspace_bytes": (S, [I64, I64]),
        "qlora_quantize_nf4_dq": (ctypes.c_int, [P, ctypes.c_int, W, P, S, P]),
        "qlora_quantize_nf4_dq_noalloc": (ctypes.c_int, [P, ctypes.c_int, W, P]),
        "qlora_dequantize_nf4_dq": (ctypes.c_int, [W, P, P]),
        "qlora_dequantize_nf4_dq_ex": (ctypes.c_int, [W, P, ctypes.c_int, P]),
        "qlora_linear_workspace_bytes": (S, [I64, I64, I64, I32]),
        "qlora_linear_fwd": (ctypes.c_int, [W, P, I64, P, P, I32, F, P, ctypes.c_int, P, P, S, P]),
        "qlora_linear_bwd": (ctypes.c_int, [W, P, P, I64, P, P, I32, F, P, P, ctypes.c_int, P, P, P, S, P]),
        "qlora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "qlora_check_device_error": (ctypes.c_int, [P]),
        "qlora_timing_enable": (ctypes.c_int, [ctypes.c_int]),
        "qlora_timing_reset": (ctypes.c_int, []),
        "qlora_timing_read": (ctypes.c_int, [P, P]),
        "qlora_launch_count": (ctypes.c_int64, []),
        "qlora_debug_inject_stall": (ctypes.c_int, [ctypes.c_int, ctypes.c_uint64]),
        "qlora_debug_bounds": (ctypes.c_int, [ctypes.c_char_p, S]),
        "qlora_debug_bounds_selftest": (ctypes.c_int, []),
        "qlora_paged_alloc": (ctypes.c_int, [S, ctypes.POINTER(ctypes.c_void_p)]),
        "qlora_paged_free": (ctypes.c_int, [P]),
        "qlora_paged_prefetch": (ctypes.c_int, [P, S, ctypes.c_int, P]),
        "qlora_adamw_step": (ctypes.c_int, [P, P, P, P, P, I64, ctypes.POINTER(qlora_adamw_hparams), P]),
        "qlora_block_workspace_bytes": (S, [ctypes.POINTER(qlora_block)]),
        "qlora_linear_workspace_bytes_ex": (S, [I64, I64, I64, I32, ctypes.POINTER(qlora_linear_opts)]),
        "qlora_linear_fwd_ex": (ctypes.c_int, [W, P, I64, P, P, I32, F, P, ctypes.c_int, P, P, S, P,
                                               ctypes.POINTER(qlora_linear_opts)]),
        "qlora_linear_bwd_ex": (ctypes.c_int, [W, P, P, I64, P, P, I32, F, P, P, ctypes.c_int, P, P, P, S, P,
                                               ctypes.POINTER(qlora_linear_opts)]),
        "qlora_linear_adapter_fwd": (ctypes.c_int, [W, P, I64, P, P, I32, F, P, P, S, P,
                                                    ctypes.POINTER(qlora_linear_opts)]),
        "qlora_linear_adapter_bwd": (ctypes.c_int, [W, P, P, I64, P, P, I32, F, P, P, S, P,
                                                    ctypes.POINTER(qlora_linear_opts)]),
        "qlora_block_fwd": (ctypes.c_int, [ctypes.POINTER(qlora_block), P, P, P, S, P]),
        "qlora_block_bwd": (ctypes.c_int, [ctypes.POINTER(qlora_block), P, P, P, P, P, P, S, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _check(status: int, where: str):
    if status != 0:
        raise QLoraError(status, where)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return QLORA_BF16
    if t.dtype == torch.float32:
        return QLORA_FP32
    if t.dtype == torch.float16:
        return QLORA_FP16
    raise TypeError(f"unsupported dtype {t.dtype}")


# ---- quantized weight container (device buffers owned by torch) ----------------

class NF4Weight:
    """Device buffers of one quantized weight plus its C descriptor."""

    def __init__(self, rows: int, cols: int, codebook=None, device="cuda"):
        if cols % QLORA_BLOCK:
            raise ValueError("cols must be a multiple of 64")
        nblocks = rows * cols // QLORA_BLOCK
        ngroups = -(-nblocks // QLORA_GROUP)
        self.rows, self.cols = rows, cols
        self.packed = torch.empty(rows * cols // 2, dtype=torch.uint8, device=device)
        self.code2 = torch.empty(nblocks, dtype=torch.uint8, device=device)
        self.c2 = torch.empty(ngroups, dtype=torch.float32, device=device)
        self.mean = torch.zeros(4, dtype=torch.float32, device=device)   # 16-byte slot, [0] used
        self.codebook = list(codebook) if codebook is not None else qlora_build_nf4_codebook()
        self.desc = qlora_nf4_weight(rows, cols, self.packed.data_ptr(), self.code2.data_ptr(),
                                     self.c2.data_ptr(), self.mean.data_ptr(),
                                     (ctypes.c_float * 16)(*self.codebook))

    @property
    def nbytes(self) -> int:
        return self.packed.numel() + self.code2.numel() + 4 * self.c2.numel() + 4


# ---- entry points (same names as the C ABI) -------------------------------------------

def qlora_build_nf4_codebook(delta: float = 0.0):
    out = (ctypes.c_float * 16)()
    _check(lib.qlora_build_nf4_codebook(delta, ctypes.cast(out, ctypes.c_void_p)), "qlora_build_nf4_codebook")
    return [float(v) for v in out]


def qlora_build_nfk_codebook(k: int, delta: float = 0.0):
    out = (ctypes.c_float * 16)()
    _check(lib.qlora_build_nfk_codebook(k, delta, ctypes.cast(out, ctypes.c_void_p)), "qlora_build_nfk_codebook")
    return [float(v) for v in out]


def qlora_build_int4_codebook():
    out = (ctypes.c_float * 16)()
    _check(lib.qlora_build_int4_codebook(ctypes.cast(out, ctypes.c_void_p)), "qlora_build_int4_codebook")
    return [float(v) for v in out]


def qlora_build_fp4_codebook():
    out = (ctypes.c_float * 16)()
    _check(lib.qlora_build_fp4_codebook(ctypes.cast(out, ctypes.c_void_p)), "qlora_build_fp4_codebook")
    return [float(v) for v in out]


def qlora_quantize_workspace_bytes(rows: int, cols: int) -> int:
    return lib.qlora_quantize_workspace_bytes(rows, cols)


def qlora_quantize_nf4_dq(W: torch.Tensor, out: NF4Weight, workspace: torch.Tensor, stream=None):
    _check(lib.qlora_quantize_nf4_dq(_ptr(W), _dtype_code(W), ctypes.byref(out.desc), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream)),
           "qlora_quantize_nf4_dq")


def qlora_quantize_nf4_dq_noalloc(W: torch.Tensor, out: NF4Weight, stream=None):
    """qlora_quantize_nf4_dq with the library's fixed scratch array instead of a
    workspace (at most QLORA_NOALLOC_MAX_BLOCKS blocks of 64; calls must not
    overlap in time)."""
    _check(lib.qlora_quantize_nf4_dq_noalloc(_ptr(W), _dtype_code(W), ctypes.byref(out.desc), _stream(stream)),
           "qlora_quantize_nf4_dq_noalloc")


def qlora_dequantize_nf4_dq(w: NF4Weight, out: torch.Tensor, stream=None):
    """bf16 output (the default compute dtype), or fp16 when `out` is fp16."""
    if out.dtype == torch.float16:
        _check(lib.qlora_dequantize_nf4_dq_ex(ctypes.byref(w.desc), _ptr(out), QLORA_FP16, _stream(stream)),
               "qlora_dequantize_nf4_dq_ex")
    else:
        _check(lib.qlora_dequantize_nf4_dq(ctypes.byref(w.desc), _ptr(out), _stream(stream)),
               "qlora_dequantize_nf4_dq")


def _opts(dropout, X, adapter_ready=False, always=False):
    """Options for the _ex calls, or None for the plain ones.  dropout: None, or
    (mask, p) with mask a uint8 device tensor of M*K/8 bytes (bit k % 8 of byte
    (m*K + k) / 8: element (m, k) kept); the compute dtype follows X (fp16
    tensors select the fp16 compute dtype); adapter_ready: the adapter's
    products were written into the workspace by the matching adapter call."""
    f16 = X is not None and X.dtype == torch.float16
    if dropout is None and not f16 and not adapter_ready and not always:
        return None
    mask, p = dropout if dropout is not None else (None, 0.0)
    return qlora_linear_opts(None if mask is None else mask.data_ptr(), p, QLORA_FP16 if f16 else QLORA_BF16,
                             1 if adapter_ready else 0)


def qlora_linear_workspace_bytes(M: int, N: int, K: int, r: int, dropout=None) -> int:
    if dropout is None:
        return lib.qlora_linear_workspace_bytes(M, N, K, r)
    o = qlora_linear_opts(1, 0.0, QLORA_BF16, 0)   # only the presence of a mask matters for the size
    return lib.qlora_linear_workspace_bytes_ex(M, N, K, r, ctypes.byref(o))


def qlora_linear_fwd(w: NF4Weight, X, M: int, A, B, r: int, scale: float, Y, H_save=None,
                     workspace=None, stream=None, dropout=None, adapter_ready=False):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = (ctypes.byref(w.desc), _ptr(X), M, _ptr(A), _ptr(B), r, scale, _ptr(Y), _dtype_code(Y), _ptr(H_save),
            _ptr(workspace), ws_bytes, _stream(stream))
    opts = _opts(dropout, X, adapter_ready)
    if opts is None:
        _check(lib.qlora_linear_fwd(*args), "qlora_linear_fwd")
    else:
        _check(lib.qlora_linear_fwd_ex(*args, ctypes.byref(opts)), "qlora_linear_fwd_ex")


def qlora_linear_bwd(w: NF4Weight, X, dY, M: int, A, B, r: int, scale: float, H_saved, dX, dA, dB,
                     workspace=None, stream=None, dropout=None, adapter_ready=False):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    dx_code = (QLORA_FP16 if X is not None and X.dtype == torch.float16 else QLORA_BF16) if dX is None \
        else _dtype_code(dX)
    args = (ctypes.byref(w.desc), _ptr(X), _ptr(dY), M, _ptr(A), _ptr(B), r, scale, _ptr(H_saved), _ptr(dX),
            dx_code, _ptr(dA), _ptr(dB), _ptr(workspace), ws_bytes, _stream(stream))
    opts = _opts(dropout, X, adapter_ready)
    if opts is None:
        _check(lib.qlora_linear_bwd(*args), "qlora_linear_bwd")
    else:
        _check(lib.qlora_linear_bwd_ex(*args, ctypes.byref(opts)), "qlora_linear_bwd_ex")


def qlora_linear_adapter_fwd(w: NF4Weight, X, M: int, A, B, r: int, scale: float, H_save=None,
                             workspace=None, stream=None, dropout=None):
    """The forward's adapter products alone (H into the workspace and H_save);
    follow with qlora_linear_fwd(..., adapter_ready=True) on the same workspace."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    opts = _opts(dropout, X, always=True)
    _check(lib.qlora_linear_adapter_fwd(ctypes.byref(w.desc), _ptr(X), M, _ptr(A), _ptr(B), r, scale, _ptr(H_save),
                                        _ptr(workspace), ws_bytes, _stream(stream), ctypes.byref(opts)),
           "qlora_linear_adapter_fwd")


def qlora_linear_adapter_bwd(w: NF4Weight, X, dY, M: int, A, B, r: int, scale: float, H_saved,
                             workspace=None, stream=None, dropout=None):
    """The backward's adapter products alone (G, and H's hi/lo halves, into the
    workspace); follow with qlora_linear_bwd(..., adapter_ready=True)."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    opts = _opts(dropout, X, always=True)
    _check(lib.qlora_linear_adapter_bwd(ctypes.byref(w.desc), _ptr(X), _ptr(dY), M, _ptr(A), _ptr(B), r, scale,
                                        _ptr(H_saved), _ptr(workspace), ws_bytes, _stream(stream),
                                        ctypes.byref(opts)),
           "qlora_linear_adapter_bwd")


def qlora_status_string(status: int) -> str:
    return lib.qlora_status_string(status).decode()


def qlora_check_device_error(stream=None):
    _check(lib.qlora_check_device_error(_stream(stream)), "qlora_check_device_error")


def qlora_timing_enable(enable: bool = True):
    _check(lib.qlora_timing_enable(1 if enable else 0), "qlora_timing_enable")


def qlora_timing_reset():
    _check(lib.qlora_timing_reset(), "qlora_timing_reset")


def qlora_timing_read() -> dict:
    """{kind: (total_ms, launches)} since the last reset (waits for the events)."""
    ms = (ctypes.c_double * len(KERNEL_KINDS))()
    n = (ctypes.c_int64 * len(KERNEL_KINDS))()
    _check(lib.qlora_timing_read(ctypes.cast(ms, ctypes.c_void_p), ctypes.cast(n, ctypes.c_void_p)),
           "qlora_timing_read")
    return {k: (ms[i], n[i]) for i, k in enumerate(KERNEL_KINDS)}


def qlora_launch_count() -> int:
    return lib.qlora_launch_count()


def qlora_debug_inject_stall(kind: str, timeout_ns: int = 1_000_000):
    """Failure-detection test hook: arms a one-shot stall in the next launch of
    kernel family `kind` ("quantize", "fwd_fused" or "bwd_fused"; None disarms)."""
    code = -1 if kind is None else KERNEL_KINDS.index(kind)
    _check(lib.qlora_debug_inject_stall(code, timeout_ns), "qlora_debug_inject_stall")


def qlora_debug_bounds_selftest():
    """Bounds-checked build only: records one failed check without touching memory."""
    _check(lib.qlora_debug_bounds_selftest(), "qlora_debug_bounds_selftest")


def qlora_debug_bounds():
    """The bounds-checked build's record: (line, source file) of the first
    failed index check since the last call, (0, "") if none; (-1, "") in the
    ordinary build."""
    buf = ctypes.create_string_buffer(128)
    line = lib.qlora_debug_bounds(buf, 128)
    return line, buf.value.decode()


# ---- paged optimizer -----------------------------------------------------------------

class PagedBuffer:
    """A unified-memory allocation from qlora_paged_alloc, viewed as a float32
    torch tensor on the current device (zero-filled).  Freed with free() or
    when the object is collected."""

    def __init__(self, numel: int, device="cuda"):
        ptr = ctypes.c_void_p()
        self.nbytes = 4 * numel
        _check(lib.qlora_paged_alloc(self.nbytes, ctypes.byref(ptr)), "qlora_paged_alloc")
        self.ptr = ptr.value
        dev = torch.device(device)
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        # a DLPack-free view: torch wraps the raw pointer without owning it
        self.tensor = _wrap_device_pointer(self.ptr, numel, dev)

    def free(self):
        if self.ptr:
            self.tensor = None
            _check(lib.qlora_paged_free(ctypes.c_void_p(self.ptr)), "qlora_paged_free")
            self.ptr = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def _wrap_device_pointer(ptr: int, numel: int, device):
    class _Arr:
        __cuda_array_interface__ = {"shape": (numel,), "typestr": "<f4", "data": (ptr, False), "version": 3,
                                    "strides": None}
    with torch.cuda.device(device):
        return torch.as_tensor(_Arr(), device=device)


def qlora_paged_prefetch(buf, to_device: bool, stream=None, nbytes=None):
    ptr = buf.ptr if isinstance(buf, PagedBuffer) else buf.data_ptr()
    n = nbytes if nbytes is not None else (buf.nbytes if isinstance(buf, PagedBuffer) else buf.numel() * buf.element_size())
    _check(lib.qlora_paged_prefetch(ctypes.c_void_p(ptr), n, 1 if to_device else 0, _stream(stream)),
           "qlora_paged_prefetch")


def qlora_adamw_step(param, param_bf16, grad, exp_avg, exp_avg_sq, lr, beta1, beta2, eps, weight_decay, step,
                     stream=None):
    h = qlora_adamw_hparams(lr, beta1, beta2, eps, weight_decay, step)
    _check(lib.qlora_adamw_step(_ptr(param), _ptr(param_bf16), _ptr(grad), _ptr(exp_avg), _ptr(exp_avg_sq),
                                param.numel(), ctypes.byref(h), _stream(stream)),
           "qlora_adamw_step")


# ---- transformer block ------------------------------------------------------------------

BLOCK_LINEARS = ("q", "k", "v", "o", "gate", "up", "down")


class Block:
    """Descriptor of one QLoRA transformer block: the seven quantized weights
    (NF4Weight, in the order of BLOCK_LINEARS), their bf16 adapters A [r][in],
    B [out][r], and the two bf16 norm weights, all device tensors kept alive
    by this object."""

    def __init__(self, batch, seq, hidden, heads, inter, r, lora_scale, weights, A, B, norm1, norm2,
                 rms_eps=1e-6, rope_base=10000.0):
        self.weights, self.A, self.B, self.norm1, self.norm2 = list(weights), list(A), list(B), norm1, norm2
        self.desc = qlora_block(batch, seq, hidden, heads, hidden // heads, inter, r, lora_scale, rms_eps,
                                rope_base, (qlora_nf4_weight * 7)(*[w.desc for w in self.weights]),
                                (ctypes.c_void_p * 7)(*[a.data_ptr() for a in self.A]),
                                (ctypes.c_void_p * 7)(*[b.data_ptr() for b in self.B]),
                                norm1.data_ptr(), norm2.data_ptr())


def qlora_block_workspace_bytes(block: Block) -> int:
    return lib.qlora_block_workspace_bytes(ctypes.byref(block.desc))


def qlora_block_fwd(block: Block, x, y, workspace, stream=None):
    _check(lib.qlora_block_fwd(ctypes.byref(block.desc), _ptr(x), _ptr(y), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream)), "qlora_block_fwd")


def qlora_block_bwd(block: Block, x, dy, dx, dA, dB, workspace, stream=None):
    pa = (ctypes.c_void_p * 7)(*[t.data_ptr() for t in dA])
    pb = (ctypes.c_void_p * 7)(*[t.data_ptr() for t in dB])
    _check(lib.qlora_block_bwd(ctypes.byref(block.desc), _ptr(x), _ptr(dy), _ptr(dx),
                               ctypes.cast(pa, ctypes.c_void_p), ctypes.cast(pb, ctypes.c_void_p), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream)), "qlora_block_bwd")
