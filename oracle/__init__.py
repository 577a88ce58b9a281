"""CPU oracle for the FP8 runtime linear path -- TEST INFRASTRUCTURE ONLY.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``fp8_dynamic_scaled_b200``) never imports it and shares no code with it.

The arithmetic lives in ``fp8_oracle.c`` (plain C, IEEE binary32 without
contraction for the fp32 steps, fp64 for the GEMM reference); this module only
builds it with gcc and marshals numpy arrays through ctypes.  The independent
NumPy nearest-code encoder in ``numpy_encoder.py`` is a second opinion used by
the pin tests.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

E4M3, E5M2 = 0, 1
TENSOR, ROW, BLOCK_1x128, BLOCK_128x128, MX32, DELAYED = 0, 1, 2, 3, 4, 5

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile fp8_oracle.c into liboracle.so with gcc (no fast-math, no FMA contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-pthread",
           "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P, I64, I32, D, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_float
    lib.orc_fmax.restype, lib.orc_fmax.argtypes = D, [I32]
    lib.orc_decode.restype, lib.orc_decode.argtypes = D, [ctypes.c_uint8, I32]
    lib.orc_encode.restype, lib.orc_encode.argtypes = ctypes.c_uint8, [D, I32]
    lib.orc_encode_bruteforce.restype = ctypes.c_uint8
    lib.orc_encode_bruteforce.argtypes = [D, I32]
    lib.orc_scale_from_amax.restype, lib.orc_scale_from_amax.argtypes = F, [F, I32]
    lib.orc_mx_exponent.restype, lib.orc_mx_exponent.argtypes = I32, [F]
    lib.orc_f32_to_bf16.restype, lib.orc_f32_to_bf16.argtypes = ctypes.c_uint16, [F]
    lib.orc_scale_count.restype, lib.orc_scale_count.argtypes = I64, [I32, I64, I64]
    lib.orc_quantize.restype = I32
    lib.orc_quantize.argtypes = [P, I64, I64, I64, I32, I32, P, P, P]
    lib.orc_delayed_step.restype = I32
    lib.orc_delayed_step.argtypes = [P, I64, I64, I64, I32, P, ctypes.c_int32, I64, P, P, P, P]
    lib.orc_gemm_ref_points.restype = I32
    lib.orc_gemm_ref_points.argtypes = [P, P, I32, I32, P, P, I32, I32, I64, I64, I64,
                                        P, P, I64, P, P]
    lib.orc_gemm_ref_full.restype = I32
    lib.orc_gemm_ref_full.argtypes = [P, P, I32, I32, P, P, I32, I32, I64, I64, I64, P, P]
    lib.orc_gemm_ref_slice.restype = I32
    lib.orc_gemm_ref_slice.argtypes = [P, P, I32, I32, P, P, I32, I32, I64, I64, I64, I64, I64, P, P]
    lib.orc_decode_table.restype, lib.orc_decode_table.argtypes = None, [I32, P]
    for name in ("orc_encode_array", "orc_encode_bruteforce_array"):
        getattr(lib, name).restype = None
        getattr(lib, name).argtypes = [P, I64, I32, P]
    lib.orc_f32_to_bf16_array.restype, lib.orc_f32_to_bf16_array.argtypes = None, [P, I64, P]
    lib.orc_quant_scaled_array.restype = None
    lib.orc_quant_scaled_array.argtypes = [P, I64, F, I32, P]
    lib.orc_dequant_scaled_array.restype = None
    lib.orc_dequant_scaled_array.argtypes = [P, I64, F, I32, P]
    lib.orc_set_threads.restype, lib.orc_set_threads.argtypes = None, [I32]
    lib.orc_get_threads.restype, lib.orc_get_threads.argtypes = I32, []
    _lib = lib
    return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


class OracleError(RuntimeError):
    pass


def set_threads(n: int) -> None:
    """Threads the oracle's array-wide functions use (rows, row blocks or output points
    split into contiguous ranges; the results do not depend on the count).  Default 1."""
    _load().orc_set_threads(int(n))


def get_threads() -> int:
    return int(_load().orc_get_threads())


class threads:
    """Context manager: run the oracle on `n` threads inside the block."""

    def __init__(self, n: int):
        self.n = int(n)

    def __enter__(self):
        self.prev = get_threads()
        set_threads(self.n)
        return self

    def __exit__(self, *exc):
        set_threads(self.prev)


def fmax(fmt: int) -> float:
    return _load().orc_fmax(fmt)


def decode(code: int, fmt: int) -> float:
    return _load().orc_decode(code, fmt)


def decode_table(fmt: int) -> np.ndarray:
    out = np.empty(256, np.float64)
    _load().orc_decode_table(fmt, _ptr(out))
    return out


def encode(values, fmt: int) -> np.ndarray:
    v = np.ascontiguousarray(values, dtype=np.float32).ravel()
    out = np.empty(v.size, np.uint8)
    _load().orc_encode_array(_ptr(v), v.size, fmt, _ptr(out))
    return out


def encode_bruteforce(values, fmt: int) -> np.ndarray:
    v = np.ascontiguousarray(values, dtype=np.float32).ravel()
    out = np.empty(v.size, np.uint8)
    _load().orc_encode_bruteforce_array(_ptr(v), v.size, fmt, _ptr(out))
    return out


def quant_scaled(values, s: float, fmt: int) -> np.ndarray:
    """Codes of fp32 values under one fp32 scale: encode(clip(fp32(x / s)))."""
    v = np.ascontiguousarray(values, dtype=np.float32).ravel()
    out = np.empty(v.size, np.uint8)
    _load().orc_quant_scaled_array(_ptr(v), v.size, float(s), fmt, _ptr(out))
    return out


def dequant_scaled(codes, s: float, fmt: int) -> np.ndarray:
    """bf16 bit patterns of fp32(decode(q) * s) ([FFS] "Scale 怎样把 Tensor 塞进 E4M3": X^ = s X_fp8)."""
    q = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(q.size, np.uint16)
    _load().orc_dequant_scaled_array(_ptr(q.ravel()), q.size, float(s), fmt, _ptr(out))
    return out.reshape(q.shape)


def f32_to_bf16(values) -> np.ndarray:
    v = np.ascontiguousarray(values, dtype=np.float32).ravel()
    out = np.empty(v.size, np.uint16)
    _load().orc_f32_to_bf16_array(_ptr(v), v.size, _ptr(out))
    return out.reshape(np.shape(values))


def scale_from_amax(amax: float, fmt: int) -> float:
    return _load().orc_scale_from_amax(amax, fmt)


def mx_exponent(amax: float) -> int:
    return _load().orc_mx_exponent(amax)


def scale_shape(mode: int, rows: int, cols: int):
    if mode in (TENSOR, DELAYED):
        return (1,)
    if mode == ROW:
        return (rows,)
    if mode == BLOCK_1x128:
        return (rows, -(-cols // 128))
    if mode == BLOCK_128x128:
        return (-(-rows // 128), -(-cols // 128))
    if mode == MX32:
        return (rows, cols // 32)
    raise ValueError(mode)


def quantize(x_bf16: np.ndarray, fmt: int, mode: int, dequant: bool = True):
    """Quantize a bf16 matrix (uint16 bit patterns, [rows, cols] or a strided view).

    Returns (codes uint8 [rows, cols], scale (float32, or uint8 E8M0 for MX32),
    dequant uint16 bf16 bits [rows, cols] or None).
    """
    assert x_bf16.dtype == np.uint16 and x_bf16.ndim == 2
    rows, cols = x_bf16.shape
    if x_bf16.strides[1] != 2 or x_bf16.strides[0] % 2 or x_bf16.strides[0] < 2 * cols:
        x_bf16 = np.ascontiguousarray(x_bf16)
    ld = x_bf16.strides[0] // 2 if rows > 0 else cols
    ptr = x_bf16.ctypes.data      # row-strided view: rows start ld elements apart
    q = np.empty((rows, cols), np.uint8)
    sdt = np.uint8 if mode == MX32 else np.float32
    scale = np.empty(scale_shape(mode, rows, cols), sdt)
    deq = np.empty((rows, cols), np.uint16) if dequant else None
    rc = _load().orc_quantize(ptr, rows, cols, ld, fmt, mode, _ptr(q), _ptr(scale), _ptr(deq))
    if rc != 0:
        raise OracleError(f"orc_quantize failed: {rc} ({'non-finite input' if rc == 1 else 'bad argument'})")
    return q, scale, deq


def bf16_to_f32(x_bf16: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns: the pattern is the top half of the fp32 one."""
    return (np.asarray(x_bf16, np.uint16).astype(np.uint32) << 16).view(np.float32)


def amax(x_bf16: np.ndarray) -> float:
    """a_max = max |x| over a bf16 tensor ([FFS] "Scale 怎样把 Tensor 塞进 E4M3", eq. a_max = max|X|);
    0 for an empty tensor.  Non-finite input is rejected, as everywhere in the oracle."""
    v = bf16_to_f32(x_bf16)
    if v.size == 0:
        return 0.0
    if not np.all(np.isfinite(v)):
        raise OracleError("non-finite input")
    return float(np.max(np.abs(v)))


def quantize_with_amax(x_bf16: np.ndarray, fmt: int, amax_value: float, dequant: bool = True):
    """Per-tensor current scaling with a given a_max (the cast phase alone):
    s = fp32(max(a_max, 1e-12f) / F_max), q = encode(clip(fp32(x / s))), X^ = bf16(fp32(decode(q) s)).
    Returns (codes [rows, cols], s float32, dequant bf16 bits or None)."""
    assert x_bf16.dtype == np.uint16 and x_bf16.ndim == 2
    s = np.float32(scale_from_amax(np.float32(amax_value), fmt))
    q = quant_scaled(bf16_to_f32(x_bf16), float(s), fmt).reshape(x_bf16.shape)
    d = dequant_scaled(q, float(s), fmt) if dequant else None
    return q, s, d


def delayed_step(x_bf16: np.ndarray, fmt: int, ring: np.ndarray, t: int, dequant: bool = False):
    """One delayed-scaling step; updates ``ring`` (float32[h]) in place.

    Returns (codes, scale float32, dequant or None, saturated element count).
    """
    assert x_bf16.dtype == np.uint16 and x_bf16.ndim == 2 and x_bf16.flags["C_CONTIGUOUS"]
    assert ring.dtype == np.float32 and ring.flags["C_CONTIGUOUS"]
    rows, cols = x_bf16.shape
    q = np.empty((rows, cols), np.uint8)
    s = np.empty(1, np.float32)
    sat = np.zeros(1, np.int64)
    deq = np.empty((rows, cols), np.uint16) if dequant else None
    rc = _load().orc_delayed_step(_ptr(x_bf16), rows, cols, cols, fmt, _ptr(ring), ring.size, t,
                                  _ptr(q), _ptr(s), _ptr(deq), _ptr(sat))
    if rc != 0:
        raise OracleError(f"orc_delayed_step failed: {rc}")
    return q, s[0], deq, int(sat[0])


def gemm_ref_full(a, sa, a_mode, fmt_a, b, sb, b_mode, fmt_b):
    """fp64 reference Y = A_deq B_deq^T and bound sum_k |terms|; a [M,K], b [N,K] codes."""
    M, K = a.shape
    N = b.shape[0]
    y = np.empty((M, N), np.float64)
    bound = np.empty((M, N), np.float64)
    rc = _load().orc_gemm_ref_full(_ptr(np.ascontiguousarray(a)), _ptr(np.ascontiguousarray(sa)),
                                   a_mode, fmt_a, _ptr(np.ascontiguousarray(b)),
                                   _ptr(np.ascontiguousarray(sb)), b_mode, fmt_b, M, N, K,
                                   _ptr(y), _ptr(bound))
    if rc != 0:
        raise OracleError("orc_gemm_ref_full failed")
    return y, bound


def gemm_ref_slice(a, sa, a_mode, fmt_a, b, sb, b_mode, fmt_b, m0: int, m1: int):
    """fp64 reference of the output rows m0..m1-1 against every row of B (the C oracle,
    rows of B split over the threads); returns (y, bound), each [m1 - m0, N]."""
    M, K = a.shape
    N = b.shape[0]
    y = np.empty((m1 - m0, N), np.float64)
    bound = np.empty((m1 - m0, N), np.float64)
    rc = _load().orc_gemm_ref_slice(_ptr(np.ascontiguousarray(a)), _ptr(np.ascontiguousarray(sa)), a_mode, fmt_a,
                                    _ptr(np.ascontiguousarray(b)), _ptr(np.ascontiguousarray(sb)), b_mode, fmt_b,
                                    M, N, K, m0, m1, _ptr(y), _ptr(bound))
    if rc != 0:
        raise OracleError("orc_gemm_ref_slice failed")
    return y, bound


def gemm_ref_points(a, sa, a_mode, fmt_a, b, sb, b_mode, fmt_b, pm, pn):
    """fp64 reference at output points (pm[i], pn[i]); returns (y, bound)."""
    M, K = a.shape
    N = b.shape[0]
    pm = np.ascontiguousarray(pm, dtype=np.int64)
    pn = np.ascontiguousarray(pn, dtype=np.int64)
    order = np.argsort(pm, kind="stable")
    y = np.empty(pm.size, np.float64)
    bound = np.empty(pm.size, np.float64)
    pm_s, pn_s = np.ascontiguousarray(pm[order]), np.ascontiguousarray(pn[order])
    ys = np.empty_like(y)
    bs = np.empty_like(bound)
    rc = _load().orc_gemm_ref_points(_ptr(np.ascontiguousarray(a)), _ptr(np.ascontiguousarray(sa)),
                                     a_mode, fmt_a, _ptr(np.ascontiguousarray(b)),
                                     _ptr(np.ascontiguousarray(sb)), b_mode, fmt_b, M, N, K,
                                     _ptr(pm_s), _ptr(pn_s), pm.size, _ptr(ys), _ptr(bs))
    if rc != 0:
        raise OracleError("orc_gemm_ref_points failed")
    y[order] = ys
    bound[order] = bs
    return y, bound


def _dequant_rows_f64(codes, scale, mode: int, fmt: int, rows: np.ndarray) -> np.ndarray:
    """S(r, k) * decode(codes[r, k]) in fp64 for the given rows r (the scale that covers
    each element, in the layouts of ``quantize``)."""
    codes = np.asarray(codes, np.uint8)
    K = codes.shape[1]
    v = decode_table(fmt)[codes[rows]]
    s = np.asarray(scale)
    if mode in (TENSOR, DELAYED):
        return v * np.float64(s.reshape(-1)[0])
    if mode == ROW:
        return v * s.reshape(-1)[rows].astype(np.float64)[:, None]
    if mode == BLOCK_1x128:
        return v * np.repeat(s[rows].astype(np.float64), 128, axis=1)[:, :K]
    if mode == BLOCK_128x128:
        return v * np.repeat(s[rows // 128].astype(np.float64), 128, axis=1)[:, :K]
    if mode == MX32:
        return v * np.repeat(np.exp2(s[rows].astype(np.float64) - 127.0), 32, axis=1)
    raise ValueError(mode)


def gemm_ref_rows(a, sa, a_mode, fmt_a, b, sb, b_mode, fmt_b, rows, chunk: int = 2048):
    """fp64 reference of whole output rows: y[i, n] = sum_k A_deq[rows[i], k] B_deq[n, k]
    and the bound sum_k |same product| ([FFS] "一次 FP8 GEMM 的完整精度契约"), for bands of
    rows of a large GEMM.  The operands are dequantised exactly in fp64 (a code times a
    power of two or an fp32 scale) and the sums run through NumPy's fp64 matmul (a
    library step), B in chunks of `chunk` rows to bound the memory."""
    rows = np.asarray(rows, np.int64)
    ad = _dequant_rows_f64(a, sa, a_mode, fmt_a, rows)
    aa = np.abs(ad)
    N = np.asarray(b).shape[0]
    y = np.empty((rows.size, N), np.float64)
    bound = np.empty((rows.size, N), np.float64)
    for n0 in range(0, N, chunk):
        n1 = min(N, n0 + chunk)
        bd = _dequant_rows_f64(b, sb, b_mode, fmt_b, np.arange(n0, n1))
        y[:, n0:n1] = ad @ bd.T
        bound[:, n0:n1] = aa @ np.abs(bd).T
    return y, bound


def epilogue_ref(y_ref, bound, bias_bf16=None):
    """GEMM reference with the output bias ([PQG] code fp8_gemm_forward: bias added to the
    scaled product before the BF16 output): y + bias[n] in fp64, and |bias[n]| added to the
    bound of the acceptance rule."""
    if bias_bf16 is None:
        return y_ref, bound
    b = bf16_to_f32(bias_bf16).astype(np.float64)
    return y_ref + b, bound + np.abs(b)


def weight_only_ref(x_bf16, w_codes, w_scale, w_mode: int, w_fmt: int):
    """Weight-only FP8 linear ([FFS] "FP8 formats, scaling and LLM inference", section
    "Weight-only FP8 与 W8A8 FP8": the weight is stored in FP8, the activation stays
    BF16): y[m, n] = sum_k x[m, k] * (s_w[n] * decode(w[n, k])) in fp64, with the
    bound sum_k |same product| of the acceptance rule.  s_w is the per-tensor or
    per-row scale of the weight's quantisation (the matmul is a library step)."""
    x = bf16_to_f32(np.asarray(x_bf16, np.uint16)).astype(np.float64)
    table = decode_table(w_fmt)
    wd = table[np.asarray(w_codes, np.uint8)]
    s = np.asarray(w_scale, np.float64).reshape(-1)
    if w_mode == ROW:
        wd = wd * s[:, None]
    elif w_mode in (TENSOR, DELAYED):
        wd = wd * s[0]
    else:
        raise ValueError("weight-only takes per-tensor or per-row weight scales")
    return x @ wd.T, np.abs(x) @ np.abs(wd).T


def requant_interval(y_ref, lim, s_y: float, fmt: int):
    """Values an FP8 output code may decode to when the bf16 output y lies within
    [y_ref - lim, y_ref + lim] and is then quantised with the fixed scale s_y
    ([FFS] "一次 FP8 GEMM 的完整精度契约": output scale / requantisation for an FP8
    consumer).  The quantiser is monotone, so the code of y lies between the codes of
    the interval's ends.  Returns the decoded values (unscaled, i.e. before the factor
    s_y) of the lowest and the highest admissible code, elementwise."""
    y_ref = np.asarray(y_ref, np.float64)
    lo = quant_scaled((y_ref - lim).astype(np.float32), s_y, fmt)
    hi = quant_scaled((y_ref + lim).astype(np.float32), s_y, fmt)
    table = decode_table(fmt)
    return table[lo].reshape(y_ref.shape), table[hi].reshape(y_ref.shape)


def bf16_ulp(y: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |y| (8 significant bits; subnormal floor 2^-133)."""
    a = np.abs(np.asarray(y, np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(a > 0, np.exp2(e - 7.0), 2.0 ** -133)


def gemm_within_tolerance(y_gpu, y_ref, bound, rel: float = 1e-3):
    """The GEMM acceptance rule: |y - y_ref| <= rel * sum_k|terms| + 1 bf16 ulp of y_ref."""
    err = np.abs(np.asarray(y_gpu, np.float64) - y_ref)
    lim = rel * bound + bf16_ulp(y_ref)
    return err <= lim, err, lim
