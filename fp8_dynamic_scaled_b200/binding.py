"""ctypes binding of libfp8.so -- argument marshalling only.

Every function here has the name of the C entry point it calls (include/fp8.h)
and does nothing but check tensor types, turn torch tensors into device
pointers and raise on a non-zero status.  All arithmetic runs in the CUDA
kernels of libfp8.so; there is no CPU or PyTorch fallback, and importing this
module fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m fp8_dynamic_scaled_b200.build` "
                      "(the FP8 path has no fallback)")

_lib = ctypes.CDLL(LIB_PATH)

# enums (include/fp8.h)
FP8_E4M3, FP8_E5M2 = 0, 1
FP8_SCALE_TENSOR, FP8_SCALE_ROW, FP8_SCALE_BLOCK_1x128 = 0, 1, 2
FP8_SCALE_BLOCK_128x128, FP8_SCALE_MX32, FP8_SCALE_DELAYED = 3, 4, 5
FP8_OK, FP8_ERR_INVALID_ARG, FP8_ERR_ALIGNMENT, FP8_ERR_UNSUPPORTED_DEVICE = 0, 1, 2, 3
FP8_ERR_NONFINITE, FP8_ERR_TIMEOUT, FP8_ERR_CUDA, FP8_ERR_WORKSPACE = 4, 5, 6, 7

EXPORTED = ("fp8_abi_version", "fp8_status_string", "fp8_device_check", "fp8_workspace_size",
            "fp8_quantize", "fp8_scaled_gemm", "fp8_linear_forward", "fp8_linear_forward_noalloc",
            "fp8_amax", "fp8_quantize_with_amax", "fp8_scaled_gemm_ex", "fp8_linear_forward_ex",
            "fp8_weight_only_linear", "fp8_testing_set_wait_limit_ns", "fp8_testing_encode_f32_range")
FP8_WEIGHT_ONLY_MAX_TOKENS = 64
FP8_NOALLOC_SCRATCH_BYTES = 4194304


class fp8_history_t(ctypes.Structure):
    _fields_ = [("ring_dev", ctypes.c_void_p), ("len", ctypes.c_int32), ("step", ctypes.c_int64),
                ("pending_dev", ctypes.c_void_p), ("ticket_dev", ctypes.c_void_p)]


class fp8_epilogue_t(ctypes.Structure):
    _fields_ = [("bias_dev", ctypes.c_void_p), ("amax_dev", ctypes.c_void_p), ("yq_dev", ctypes.c_void_p),
                ("yq_scale_dev", ctypes.c_void_p), ("yq_fmt", ctypes.c_int32), ("ldq", ctypes.c_int64)]


_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_lib.fp8_abi_version.restype, _lib.fp8_abi_version.argtypes = _I32, []
_lib.fp8_status_string.restype, _lib.fp8_status_string.argtypes = ctypes.c_char_p, [_I32]
_lib.fp8_device_check.restype, _lib.fp8_device_check.argtypes = _I32, []
_lib.fp8_workspace_size.restype = _SZ
_lib.fp8_workspace_size.argtypes = [_I32, _I64, _I64, _I64, _I32]
_lib.fp8_quantize.restype = _I32
_lib.fp8_quantize.argtypes = [_P, _I64, _I64, _I64, _I32, _I32, _P, _P, ctypes.POINTER(fp8_history_t), _P, _P,
                              _P, _SZ, _P]
_lib.fp8_scaled_gemm.restype = _I32
_lib.fp8_scaled_gemm.argtypes = [_P, _P, _I32, _I32, _P, _P, _I32, _I32, _I64, _I64, _I64, _P, _I64, _P, _P,
                                 _SZ, _P]
_lib.fp8_linear_forward.restype = _I32
_lib.fp8_linear_forward.argtypes = [_P, _I64, _I64, _I64, _I32, _I32, ctypes.POINTER(fp8_history_t), _P, _P,
                                    _I32, _I32, _I64, _P, _I64, _P, _P, _SZ, _P]
_lib.fp8_amax.restype = _I32
_lib.fp8_amax.argtypes = [_P, _I64, _I64, _I64, _P, _P, _P, _SZ, _P]
_lib.fp8_quantize_with_amax.restype = _I32
_lib.fp8_quantize_with_amax.argtypes = [_P, _I64, _I64, _I64, _I32, _P, _P, _P, _P, _P, _P]
_lib.fp8_scaled_gemm_ex.restype = _I32
_lib.fp8_scaled_gemm_ex.argtypes = [_P, _P, _I32, _I32, _P, _P, _I32, _I32, _I64, _I64, _I64, _P, _I64,
                                    ctypes.POINTER(fp8_epilogue_t), _P, _P, _SZ, _P]
_lib.fp8_linear_forward_ex.restype = _I32
_lib.fp8_linear_forward_ex.argtypes = [_P, _I64, _I64, _I64, _I32, _I32, ctypes.POINTER(fp8_history_t), _P, _P,
                                       _I32, _I32, _I64, _P, _I64, ctypes.POINTER(fp8_epilogue_t), _P, _P, _SZ,
                                       _P]
_lib.fp8_weight_only_linear.restype = _I32
_lib.fp8_weight_only_linear.argtypes = [_P, _I64, _I64, _I64, _P, _P, _I32, _I32, _I64, _P, _I64, _P, _P]
_lib.fp8_testing_set_wait_limit_ns.restype = None
_lib.fp8_testing_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
_lib.fp8_testing_encode_f32_range.restype = _I32
_lib.fp8_testing_encode_f32_range.argtypes = [ctypes.c_uint32, _I64, _I32, _P, _P]
_lib.fp8_linear_forward_noalloc.restype = _I32
_lib.fp8_linear_forward_noalloc.argtypes = [_P, _I64, _I64, _I64, _I32, _I32, ctypes.POINTER(fp8_history_t), _P,
                                            _P, _I32, _I32, _I64, _P, _I64, _P, _P]


class FP8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {fp8_status_string(status)} ({status})")
        self.status = status


def _check(rc: int, where: str):
    if rc != FP8_OK:
        raise FP8Error(rc, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


# ------------------------------------------------------------------ entry points
def fp8_abi_version() -> int:
    return _lib.fp8_abi_version()


def fp8_status_string(status: int) -> str:
    return _lib.fp8_status_string(status).decode()


def fp8_device_check() -> int:
    return _lib.fp8_device_check()


def fp8_testing_set_wait_limit_ns(ns: int) -> None:
    """Testing hook (include/fp8_testing.h): limit of each GEMM pipeline wait; 0 = default."""
    _lib.fp8_testing_set_wait_limit_ns(int(ns))


def fp8_testing_encode_f32_range(first_bits: int, q, fmt: int, *, stream=None) -> None:
    """Testing hook (include/fp8_testing.h): q[i] = encode step of the fp32 value with bit
    pattern first_bits + i, for every byte of the uint8 device tensor q."""
    if q.dtype != torch.uint8 or not q.is_contiguous():
        raise TypeError("q must be a contiguous uint8 tensor")
    _check(_lib.fp8_testing_encode_f32_range(int(first_bits), q.numel(), fmt, _ptr(q), _stream(stream)),
           "fp8_testing_encode_f32_range")


def fp8_workspace_size(which: int, M: int, N: int, K: int, mode: int) -> int:
    return _lib.fp8_workspace_size(which, M, N, K, mode)


class History:
    """Device state of delayed scaling: ring[len], pending, ticket (all zero at step 0)."""

    def __init__(self, length: int = 16, device="cuda"):
        self.ring = torch.zeros(length, dtype=torch.float32, device=device)
        self.pending = torch.zeros(1, dtype=torch.float32, device=device)
        self.ticket = torch.zeros(1, dtype=torch.int32, device=device)
        self.c = fp8_history_t(self.ring.data_ptr(), length, 0, self.pending.data_ptr(), self.ticket.data_ptr())

    @property
    def step(self) -> int:
        return self.c.step


def fp8_quantize(x, fmt, mode, q, scale, *, hist: History | None = None, dequant=None, dev_status=None,
                 workspace=None, stream=None):
    """Quantize bf16 x [rows, cols] (row stride x.stride(0)) into q, scale (and dequant)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or (x.numel() and x.stride(1) != 1):
        raise TypeError("x must be a 2-D bf16 tensor with unit column stride")
    if q.dtype != torch.uint8:
        raise TypeError("q must be uint8")
    rows, cols = x.shape
    ld = x.stride(0) if rows > 1 else cols
    rc = _lib.fp8_quantize(_ptr(x), rows, cols, ld, fmt, mode, _ptr(q), _ptr(scale),
                           ctypes.byref(hist.c) if hist is not None else None, _ptr(dequant), _ptr(dev_status),
                           _ptr(workspace), _nbytes(workspace), _stream(stream))
    _check(rc, "fp8_quantize")


def fp8_scaled_gemm(a, a_scale, a_mode, fmt_a, b, b_scale, b_mode, fmt_b, y, *, dev_status=None,
                    workspace=None, stream=None):
    """y[M, N] (bf16, row stride y.stride(0)) = scaled a[M, K] . b[N, K]^T."""
    if a.dtype != torch.uint8 or b.dtype != torch.uint8 or y.dtype != torch.bfloat16:
        raise TypeError("a, b must be uint8 codes and y bf16")
    M, K = a.shape
    N = b.shape[0]
    ldy = y.stride(0) if y.shape[0] > 1 else y.shape[1]
    rc = _lib.fp8_scaled_gemm(_ptr(a), _ptr(a_scale), a_mode, fmt_a, _ptr(b), _ptr(b_scale), b_mode, fmt_b,
                              M, N, K, _ptr(y), ldy, _ptr(dev_status), _ptr(workspace), _nbytes(workspace),
                              _stream(stream))
    _check(rc, "fp8_scaled_gemm")


def fp8_linear_forward(x, x_fmt, x_mode, w, w_scale, w_mode, w_fmt, y, workspace, *, hist: History | None = None,
                       dev_status=None, stream=None):
    """y = FP8 linear(x): quantize x with x_mode into the workspace, then the scaled GEMM with w."""
    if x.dtype != torch.bfloat16 or w.dtype != torch.uint8 or y.dtype != torch.bfloat16:
        raise TypeError("x bf16, w uint8 codes, y bf16")
    M, K = x.shape
    N = w.shape[0]
    ldx = x.stride(0) if M > 1 else K
    ldy = y.stride(0) if y.shape[0] > 1 else y.shape[1]
    rc = _lib.fp8_linear_forward(_ptr(x), M, K, ldx, x_fmt, x_mode,
                                 ctypes.byref(hist.c) if hist is not None else None, _ptr(w), _ptr(w_scale),
                                 w_mode, w_fmt, N, _ptr(y), ldy, _ptr(dev_status), _ptr(workspace),
                                 _nbytes(workspace), _stream(stream))
    _check(rc, "fp8_linear_forward")


def fp8_amax(x, amax, *, dev_status=None, workspace=None, stream=None):
    """amax[0] (device fp32) = max |x| over bf16 x [rows, cols]."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or (x.numel() and x.stride(1) != 1):
        raise TypeError("x must be a 2-D bf16 tensor with unit column stride")
    rows, cols = x.shape
    ld = x.stride(0) if rows > 1 else cols
    rc = _lib.fp8_amax(_ptr(x), rows, cols, ld, _ptr(amax), _ptr(dev_status), _ptr(workspace), _nbytes(workspace),
                       _stream(stream))
    _check(rc, "fp8_amax")


def fp8_quantize_with_amax(x, fmt, amax, q, scale, *, dequant=None, dev_status=None, stream=None):
    """Per-tensor cast of bf16 x with the scale of a given device amax: scale[0] = max(amax, 1e-12)/F_max."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or (x.numel() and x.stride(1) != 1):
        raise TypeError("x must be a 2-D bf16 tensor with unit column stride")
    if q.dtype != torch.uint8:
        raise TypeError("q must be uint8")
    rows, cols = x.shape
    ld = x.stride(0) if rows > 1 else cols
    rc = _lib.fp8_quantize_with_amax(_ptr(x), rows, cols, ld, fmt, _ptr(amax), _ptr(q), _ptr(scale), _ptr(dequant),
                                     _ptr(dev_status), _stream(stream))
    _check(rc, "fp8_quantize_with_amax")


def _epilogue(N, bias, amax, yq, yq_scale, yq_fmt):
    if bias is None and amax is None and yq is None:
        return None
    if bias is not None and (bias.dtype != torch.bfloat16 or bias.numel() != N):
        raise TypeError("bias must be bf16 [N]")
    ldq = 0
    if yq is not None:
        if yq.dtype != torch.uint8:
            raise TypeError("yq must be uint8 codes")
        ldq = yq.stride(0) if yq.shape[0] > 1 else yq.shape[1]
    return fp8_epilogue_t(_ptr(bias), _ptr(amax), _ptr(yq), _ptr(yq_scale), yq_fmt, ldq)


def fp8_scaled_gemm_ex(a, a_scale, a_mode, fmt_a, b, b_scale, b_mode, fmt_b, y, *, bias=None, amax=None, yq=None,
                       yq_scale=None, yq_fmt=FP8_E4M3, dev_status=None, workspace=None, stream=None):
    """fp8_scaled_gemm with the epilogue options: bias [N] (bf16), amax (device fp32, max |y| folded in),
    yq [M, N] FP8 codes of y / yq_scale.  y may be None when yq is given."""
    if a.dtype != torch.uint8 or b.dtype != torch.uint8 or (y is not None and y.dtype != torch.bfloat16):
        raise TypeError("a, b must be uint8 codes and y bf16")
    M, K = a.shape
    N = b.shape[0]
    ldy = 0 if y is None else (y.stride(0) if y.shape[0] > 1 else y.shape[1])
    epi = _epilogue(N, bias, amax, yq, yq_scale, yq_fmt)
    rc = _lib.fp8_scaled_gemm_ex(_ptr(a), _ptr(a_scale), a_mode, fmt_a, _ptr(b), _ptr(b_scale), b_mode, fmt_b,
                                 M, N, K, _ptr(y), ldy, ctypes.byref(epi) if epi is not None else None,
                                 _ptr(dev_status), _ptr(workspace), _nbytes(workspace), _stream(stream))
    _check(rc, "fp8_scaled_gemm_ex")


def fp8_linear_forward_ex(x, x_fmt, x_mode, w, w_scale, w_mode, w_fmt, y, workspace, *, hist: History | None = None,
                          bias=None, amax=None, yq=None, yq_scale=None, yq_fmt=FP8_E4M3, dev_status=None,
                          stream=None):
    """fp8_linear_forward with the epilogue options of fp8_scaled_gemm_ex."""
    if x.dtype != torch.bfloat16 or w.dtype != torch.uint8 or (y is not None and y.dtype != torch.bfloat16):
        raise TypeError("x bf16, w uint8 codes, y bf16")
    M, K = x.shape
    N = w.shape[0]
    ldx = x.stride(0) if M > 1 else K
    ldy = 0 if y is None else (y.stride(0) if y.shape[0] > 1 else y.shape[1])
    epi = _epilogue(N, bias, amax, yq, yq_scale, yq_fmt)
    rc = _lib.fp8_linear_forward_ex(_ptr(x), M, K, ldx, x_fmt, x_mode,
                                    ctypes.byref(hist.c) if hist is not None else None, _ptr(w), _ptr(w_scale),
                                    w_mode, w_fmt, N, _ptr(y), ldy, ctypes.byref(epi) if epi is not None else None,
                                    _ptr(dev_status), _ptr(workspace), _nbytes(workspace), _stream(stream))
    _check(rc, "fp8_linear_forward_ex")


def fp8_weight_only_linear(x, w, w_scale, w_mode, w_fmt, y, *, dev_status=None, stream=None):
    """y [M, N] bf16 = x [M, K] bf16 times the FP8 weight w [N, K] (codes) with its scale."""
    if x.dtype != torch.bfloat16 or w.dtype != torch.uint8 or y.dtype != torch.bfloat16:
        raise TypeError("x bf16, w uint8 codes, y bf16")
    M, K = x.shape
    N = w.shape[0]
    ldx = x.stride(0) if M > 1 else K
    ldy = y.stride(0) if y.shape[0] > 1 else y.shape[1]
    rc = _lib.fp8_weight_only_linear(_ptr(x), M, K, ldx, _ptr(w), _ptr(w_scale), w_mode, w_fmt, N, _ptr(y), ldy,
                                     _ptr(dev_status), _stream(stream))
    _check(rc, "fp8_weight_only_linear")


def fp8_linear_forward_noalloc(x, x_fmt, x_mode, w, w_scale, w_mode, w_fmt, y, *, hist: History | None = None,
                               dev_status=None, stream=None):
    """fp8_linear_forward without a workspace argument, for callers that cannot allocate:
    the scratch is the library's fixed FP8_NOALLOC_SCRATCH_BYTES device array, shared by
    all calls (order overlapping calls on one stream)."""
    if x.dtype != torch.bfloat16 or w.dtype != torch.uint8 or y.dtype != torch.bfloat16:
        raise TypeError("x bf16, w uint8 codes, y bf16")
    M, K = x.shape
    N = w.shape[0]
    ldx = x.stride(0) if M > 1 else K
    ldy = y.stride(0) if y.shape[0] > 1 else y.shape[1]
    rc = _lib.fp8_linear_forward_noalloc(_ptr(x), M, K, ldx, x_fmt, x_mode,
                                         ctypes.byref(hist.c) if hist is not None else None, _ptr(w),
                                         _ptr(w_scale), w_mode, w_fmt, N, _ptr(y), ldy, _ptr(dev_status),
                                         _stream(stream))
    _check(rc, "fp8_linear_forward_noalloc")


# ------------------------------------------------------------------ allocation helpers
def scale_shape(mode: int, rows: int, cols: int):
    if mode in (FP8_SCALE_TENSOR, FP8_SCALE_DELAYED):
        return (1,)
    if mode == FP8_SCALE_ROW:
        return (rows,)
    if mode == FP8_SCALE_BLOCK_1x128:
        return (rows, -(-cols // 128))
    if mode == FP8_SCALE_BLOCK_128x128:
        return (-(-rows // 128), -(-cols // 128))
    if mode == FP8_SCALE_MX32:
        return (rows, cols // 32)
    raise ValueError(mode)


def empty_quant_outputs(rows: int, cols: int, mode: int, device="cuda", dequant: bool = False):
    """Output buffers of fp8_quantize for a [rows, cols] input: (q, scale, dequant or None)."""
    q = torch.empty((rows, cols), dtype=torch.uint8, device=device)
    sdt = torch.uint8 if mode == FP8_SCALE_MX32 else torch.float32
    s = torch.empty(scale_shape(mode, rows, cols), dtype=sdt, device=device)
    d = torch.empty((rows, cols), dtype=torch.bfloat16, device=device) if dequant else None
    return q, s, d


def workspace_for(which: int, M: int, N: int, K: int, mode: int, device="cuda"):
    n = fp8_workspace_size(which, M, N, K, mode)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device)
