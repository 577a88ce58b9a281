"""Seeded synthetic inputs for the FP8 runtime linear path.

This module only draws random numbers and rounds them to bf16; it holds none of
the quantisation or GEMM arithmetic.  Both the CUDA path (through the tests and
the benchmark) and the CPU oracle take their inputs from here, so the two
always see the same bits.

Workloads (sizes and value distributions):
  * ``linear_small``      X [128, 256] ~ N(0,1) with one element set to 400.0,
                          W [256, 256] ~ N(0, 0.02).
  * ``quant_sweep``       64 Mi elements ([8192, 8192]) with |x| = 10^U(-6, 4),
                          random signs, round(1e-4 * n) outliers at +-1e5.
  * ``llama70b_prefill``  X [4096, 8192] ~ N(0,1) with 0.1% of the channels (8)
                          scaled x50, W [28672, 8192] ~ N(0, 0.02).  The decode
                          shape is the same recipe with M = 16 (1 to 64 tokens in
                          the decode tests).
  * ``block_scaled``      X [8192, 8192] and W [28672, 8192]; value = N(0,1) times
                          one lognormal(0,1) draw per scaling block (1x128 for X,
                          128x128 for W).
  * ``mx_delayed``        X [16384, 8192] ~ N(0,1), W [8192, 8192] ~ N(0, 0.02);
                          the delayed sequence has X_t ~ N(0, (1 + 3t/15)^2), t = 0..15.

The seed is 42 (the pages' experiments fix SEED = 42); every tensor draws from
its own sub-stream, so shapes can be shrunk for tests without changing the
recipe.
"""
from __future__ import annotations

import numpy as np

SEED = 42

# Sub-stream identifiers: one independent PCG64 stream per tensor role.
_STREAMS = {
    "linear_small.x": 1, "linear_small.w": 2, "linear_small.outlier": 3,
    "quant_sweep.mag": 10, "quant_sweep.sign": 11, "quant_sweep.outlier": 12,
    "llama70b_prefill.x": 20, "llama70b_prefill.w": 21, "llama70b_prefill.channels": 22,
    "block_scaled.x": 30, "block_scaled.w": 31, "block_scaled.xblk": 32, "block_scaled.wblk": 33,
    "mx_delayed.x": 40, "mx_delayed.w": 41, "mx_delayed.step": 42,
}

CONFIG_SHAPES = {
    "linear_small": dict(M=128, K=256, N=256),
    "quant_sweep": dict(rows=8192, cols=8192),
    "llama70b_prefill": dict(M=4096, K=8192, N=28672),
    "block_scaled": dict(M=8192, K=8192, N=28672),
    "mx_delayed": dict(M=16384, K=8192, N=8192, steps=16, history=16),
}


def rng(stream: str, extra: int = 0, seed: int = SEED) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, _STREAMS[stream], extra]))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even) and return the uint16 bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    kept = (u >> np.uint32(16)).astype(np.uint32)
    dropped = u & np.uint32(0xFFFF)
    up = (dropped > 0x8000) | ((dropped == 0x8000) & ((kept & 1) == 1))
    kept = kept + up.astype(np.uint32)
    nan = np.isnan(f)
    if nan.any():
        kept = np.where(nan, (u >> np.uint32(16)) | np.uint32(0x40), kept)
    return kept.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(stream: str, shape, std: float = 1.0, extra: int = 0) -> np.ndarray:
    g = rng(stream, extra)
    out = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


# ---------------------------------------------------------------- workloads
def linear_small(M=128, K=256, N=256):
    """X with one planted 400.0 (the per-tensor outlier case); W ~ N(0, 0.02)."""
    x = _normal("linear_small.x", (M, K))
    g = rng("linear_small.outlier")
    idx = int(g.integers(0, M * K))
    x.reshape(-1)[idx] = 400.0
    w = _normal("linear_small.w", (N, K), std=0.02)
    return bf16_bits(x), bf16_bits(w)


def quant_sweep(rows=8192, cols=8192):
    """Log-uniform magnitudes over [1e-6, 1e4], random signs, 1e-4 of entries at +-1e5."""
    n = rows * cols
    mag = np.power(np.float32(10.0),
                   rng("quant_sweep.mag").uniform(-6.0, 4.0, size=n).astype(np.float32))
    sign = rng("quant_sweep.sign").integers(0, 2, size=n, dtype=np.int8)
    x = np.where(sign == 1, -mag, mag).astype(np.float32)
    n_out = int(round(1e-4 * n))
    g = rng("quant_sweep.outlier")
    pos = g.choice(n, size=n_out, replace=False) if n_out else np.empty(0, np.int64)
    osign = g.integers(0, 2, size=n_out)
    x[pos] = np.where(osign == 1, -1e5, 1e5).astype(np.float32)
    return bf16_bits(x.reshape(rows, cols))


def llama70b_prefill(M=4096, K=8192, N=28672, with_w=True):
    """X ~ N(0,1) with round(0.001*K) seeded channels scaled x50; W ~ N(0, 0.02)."""
    x = _normal("llama70b_prefill.x", (M, K))
    n_ch = max(1, int(0.001 * K))
    ch = rng("llama70b_prefill.channels").choice(K, size=n_ch, replace=False)
    x[:, ch] *= np.float32(50.0)
    xb = bf16_bits(x)
    wb = bf16_bits(_normal("llama70b_prefill.w", (N, K), std=0.02)) if with_w else None
    return xb, wb


def block_scaled(M=8192, K=8192, N=28672, with_w=True):
    """N(0,1) values times one lognormal(0,1) factor per 1x128 (X) / 128x128 (W) block."""
    x = _normal("block_scaled.x", (M, K))
    kb = -(-K // 128)
    fx = np.exp(rng("block_scaled.xblk").standard_normal(size=(M, kb))).astype(np.float32)
    x *= np.repeat(fx, 128, axis=1)[:, :K]
    xb = bf16_bits(x)
    wb = None
    if with_w:
        w = _normal("block_scaled.w", (N, K))
        nb = -(-N // 128)
        fw = np.exp(rng("block_scaled.wblk").standard_normal(size=(nb, kb))).astype(np.float32)
        w *= np.repeat(np.repeat(fw, 128, axis=0), 128, axis=1)[:N, :K]
        wb = bf16_bits(w)
    return xb, wb


def mx_delayed(M=16384, K=8192, N=8192, with_w=True):
    """X ~ N(0,1), W ~ N(0, 0.02) for the MXFP8 GEMM."""
    xb = bf16_bits(_normal("mx_delayed.x", (M, K)))
    wb = bf16_bits(_normal("mx_delayed.w", (N, K), std=0.02)) if with_w else None
    return xb, wb


def delayed_std(t: int, steps: int = 16) -> float:
    """Standard deviation of step t of the drifting sequence: 1 -> 4 over the steps."""
    return 1.0 + 3.0 * t / (steps - 1)


def delayed_step_input(t: int, M=16384, K=8192, steps: int = 16, base: np.ndarray | None = None):
    """X_t ~ N(0, std_t^2): a fresh draw per step (stream extra = t), or, when ``base``
    (a float32 N(0,1) draw) is given, that draw scaled by std_t."""
    std = np.float32(delayed_std(t, steps))
    if base is None:
        return bf16_bits(_normal("mx_delayed.step", (M, K), extra=t) * std)
    return bf16_bits(base * std)


def delayed_base(M=16384, K=8192) -> np.ndarray:
    return _normal("mx_delayed.step", (M, K), extra=1000)
