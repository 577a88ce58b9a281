"""Independent NumPy nearest-code encoder -- TEST INFRASTRUCTURE ONLY (a second
opinion on the C oracle's encoder, used by the pin tests).

The value table is built directly from the bit layouts stated on
"FP8 formats, scaling and LLM inference" (section "8 个 Bit 怎样分配": E4M3 is
1 sign + 4 exponent + 3 mantissa bits, E5M2 is 1 + 5 + 2) with the biases of
"FP8 推理：8 位浮点量化、E4M3/E5M2 与 NVIDIA FP8 生态" (section "数值特性":
bias 7 / 15).  Encoding searches the whole table for the nearest finite value
(ties to the even code) with vectorised NumPy, sharing nothing with
fp8_oracle.c.
"""
from __future__ import annotations

import numpy as np


def value_table(fmt: int) -> np.ndarray:
    """Real value of each of the 256 codes (NaN for NaN codes, +-inf for Inf codes)."""
    ebits, mbits, bias = (4, 3, 7) if fmt == 0 else (5, 2, 15)
    codes = np.arange(256)
    sign = np.where(codes >= 128, -1.0, 1.0)
    e = (codes >> mbits) & ((1 << ebits) - 1)
    m = codes & ((1 << mbits) - 1)
    frac = m / float(1 << mbits)
    vals = np.where(e == 0, frac * 2.0 ** (1 - bias), (1.0 + frac) * np.exp2(e - bias))
    vals = sign * vals
    top = (1 << ebits) - 1
    if fmt == 0:   # E4M3 "fn": only S.1111.111 is special (NaN)
        vals = np.where((e == top) & (m == (1 << mbits) - 1), np.nan, vals)
    else:          # E5M2: S.11111.00 is Inf, S.11111.xx (xx != 0) NaN
        vals = np.where((e == top) & (m == 0), sign * np.inf, vals)
        vals = np.where((e == top) & (m != 0), np.nan, vals)
    return vals


def encode_nearest(values, fmt: int, chunk: int = 1 << 16) -> np.ndarray:
    """Nearest finite code with the input's sign; exact ties go to the even code."""
    v = np.asarray(values, np.float64).ravel()
    table = value_table(fmt)
    out = np.empty(v.size, np.uint8)
    pos_codes = np.arange(128)
    pos_vals = table[:128]
    finite = np.isfinite(pos_vals)
    cand_codes = pos_codes[finite]
    cand_vals = pos_vals[finite]
    for i in range(0, v.size, chunk):
        blk = v[i:i + chunk]
        a = np.abs(blk)
        d = np.abs(a[:, None] - cand_vals[None, :])
        dmin = d.min(axis=1, keepdims=True)
        tie = d == dmin
        # among the tied candidates prefer an even code, else the lowest
        even = tie & (cand_codes[None, :] % 2 == 0)
        pick = np.where(even.any(axis=1), np.argmax(even, axis=1), np.argmax(tie, axis=1))
        mag = cand_codes[pick]
        out[i:i + chunk] = (mag | np.where(np.signbit(blk), 128, 0)).astype(np.uint8)
    return out
