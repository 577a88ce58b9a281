"""Pins for the oracle functions behind the split per-tensor scaling (amax, cast with a
given amax) and the GEMM epilogue options (bias, FP8 output codes).  Each test
checks them against numbers on the pages (tests/golden), closed forms, exact
integer arithmetic or brute force.  Runs without a GPU."""
import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden
from fp8_dynamic_scaled_b200 import inputs

E4M3, E5M2 = oracle.E4M3, oracle.E5M2


def _golden_outlier():
    rows, table = read_golden("ffs_outlier_example.txt")
    x = np.array([float(r[0]) for r in table], np.float32)
    return rows, table, x


# ------------------------------------------------------------ amax
def test_amax_outlier_example():
    """[FFS] "Per-tensor Scaling 的优点与问题": body about 1, one outlier of 400 -> a_max = 400."""
    rows, _, x = _golden_outlier()
    g = np.random.default_rng(5)
    body = np.clip(g.standard_normal((16, 64)), -1.0, 1.0).astype(np.float32)
    body[3, 17] = x[0]
    assert oracle.amax(inputs.bf16_bits(body)) == float(rows["outlier"][0])
    assert oracle.amax(inputs.bf16_bits(-body)) == float(rows["outlier"][0])


def test_amax_edge_cases_and_torch():
    assert oracle.amax(np.zeros((0, 16), np.uint16)) == 0.0
    assert oracle.amax(np.zeros((3, 16), np.uint16)) == 0.0
    # the largest finite bf16 and the smallest subnormal survive exactly
    assert oracle.amax(np.array([[0x7F7F, 0x0001]], np.uint16)) == float(np.float32(3.3895314e38))
    assert oracle.amax(np.array([[0x0001, 0x8001]], np.uint16)) == 2.0 ** -133
    with pytest.raises(oracle.OracleError):
        oracle.amax(np.array([[0x3F80, 0x7FC0]], np.uint16))
    # a library third opinion on random data
    g = np.random.default_rng(11)
    x = inputs.bf16_bits((g.standard_normal((37, 96)) * np.exp(g.standard_normal((37, 1)) * 4)).astype(np.float32))
    t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).float().abs().max().item()
    assert oracle.amax(x) == t


# ------------------------------------------------------------ cast with a given amax
def test_quantize_with_amax_outlier_golden():
    """The printed outlier example through the given-amax cast: s = fp32(400/448) and the codes."""
    rows, table, x = _golden_outlier()
    q, s, _ = oracle.quantize_with_amax(inputs.bf16_bits(x.reshape(1, -1)), E4M3, float(rows["outlier"][0]),
                                        dequant=False)
    assert s == np.float32(np.float32(400.0) / np.float32(448.0))
    assert list(q[0]) == [int(r[1], 16) for r in table]


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_quantize_with_true_amax_equals_tensor_mode(fmt):
    """With a_max = max|x| the split path is per-tensor current scaling, bit for bit."""
    g = np.random.default_rng(17 + fmt)
    x = inputs.bf16_bits((g.standard_normal((33, 160)) * 7).astype(np.float32))
    q1, s1, d1 = oracle.quantize(x, fmt, oracle.TENSOR)
    q2, s2, d2 = oracle.quantize_with_amax(x, fmt, oracle.amax(x))
    assert s1[0] == s2 and np.array_equal(q1, q2) and np.array_equal(d1, d2)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_quantize_with_small_amax_saturates(fmt):
    """A given a_max below the data's: every |x| with x/s beyond F_max lands on +-F_max,
    the rest are the plain encodings of x/s (checked against brute force)."""
    g = np.random.default_rng(23 + fmt)
    xf = (g.standard_normal((8, 64)) * 3).astype(np.float32)
    x = inputs.bf16_bits(xf)
    xv = oracle.bf16_to_f32(x)
    a = oracle.amax(x) / 4
    q, s, _ = oracle.quantize_with_amax(x, fmt, a, dequant=False)
    fm = oracle.fmax(fmt)
    t = (xv.astype(np.float32) / np.float32(s)).astype(np.float32)
    big = np.abs(t) > fm
    assert big.any() and (~big).any()
    table = oracle.decode_table(fmt)
    assert np.all(table[q[big]] == np.sign(xv[big]) * fm)
    assert np.array_equal(q[~big], oracle.encode_bruteforce(t[~big], fmt))


def test_quantize_with_amax_zero_floor():
    q, s, d = oracle.quantize_with_amax(np.zeros((2, 16), np.uint16), E4M3, 0.0)
    assert s == np.float32(np.float32(1e-12) / np.float32(448.0)) and not q.any() and not d.any()


# ------------------------------------------------------------ epilogue reference
def _codes_of(ints, fmt):
    return oracle.encode(np.asarray(ints, np.float32), fmt).reshape(np.shape(ints))


def test_epilogue_bias_exact_integer():
    """Small-integer codes, unit scales, integer bias: y + bias is an exact int64 result."""
    g = np.random.default_rng(31)
    M, N, K = 9, 24, 64
    a_int = g.integers(-6, 7, (M, K))
    b_int = g.integers(-6, 7, (N, K))
    bias_int = g.integers(-100, 101, N)
    one = np.ones(1, np.float32)
    y, bound = oracle.gemm_ref_full(_codes_of(a_int, E4M3), one, oracle.TENSOR, E4M3, _codes_of(b_int, E4M3), one,
                                    oracle.TENSOR, E4M3)
    yb, bb = oracle.epilogue_ref(y, bound, inputs.bf16_bits(bias_int.astype(np.float32)))
    assert np.array_equal(yb, (a_int @ b_int.T + bias_int[None, :]).astype(np.float64))
    assert np.array_equal(bb, (np.abs(a_int) @ np.abs(b_int).T + np.abs(bias_int)[None, :]).astype(np.float64))
    assert oracle.epilogue_ref(y, bound, None)[0] is y


def test_requant_interval_degenerate_is_the_golden_codes():
    """A zero-width interval gives the one code of y / s_y: the outlier example again."""
    rows, table, x = _golden_outlier()
    s = oracle.scale_from_amax(float(rows["outlier"][0]), E4M3)
    lo, hi = oracle.requant_interval(x.astype(np.float64), 0.0, s, E4M3)
    assert np.array_equal(lo, hi)
    assert list(lo) == [float(r[2]) for r in table]


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_requant_interval_brackets_every_value_in_range(fmt):
    """Brute force: any fp32 value within [y - lim, y + lim] quantises to a code whose
    value lies in the interval's [lo, hi]."""
    g = np.random.default_rng(41 + fmt)
    y = g.standard_normal(2000) * 50
    lim = np.abs(g.standard_normal(2000)) * 2
    s = oracle.scale_from_amax(float(np.max(np.abs(y))) / 2, fmt)   # some outputs saturate
    lo, hi = oracle.requant_interval(y, lim, s, fmt)
    table = oracle.decode_table(fmt)
    for frac in np.linspace(-1.0, 1.0, 9):
        v = (y + frac * lim).astype(np.float32)
        inside = (v >= y - lim) & (v <= y + lim)
        c = table[oracle.quant_scaled(v, s, fmt)]
        assert np.all((c[inside] >= lo[inside]) & (c[inside] <= hi[inside]))
    assert np.all(lo <= hi)


# ------------------------------------------------------------ weight-only reference
def test_weight_only_exact_integer():
    """Integer activations (exact in bf16), small-integer codes, unit scale: an int64 matmul."""
    g = np.random.default_rng(51)
    M, N, K = 5, 40, 96
    x_int = g.integers(-20, 21, (M, K))
    w_int = g.integers(-6, 7, (N, K))
    codes = _codes_of(w_int, E4M3)
    y, bound = oracle.weight_only_ref(inputs.bf16_bits(x_int.astype(np.float32)), codes, np.ones(1, np.float32),
                                      oracle.TENSOR, E4M3)
    assert np.array_equal(y, (x_int @ w_int.T).astype(np.float64))
    assert np.array_equal(bound, (np.abs(x_int) @ np.abs(w_int).T).astype(np.float64))


def test_weight_only_identity_and_row_scales():
    """W = identity codes with per-row scales s: y[m, n] = x[m, n] * s[n]; and the per-row
    reference equals a per-tensor one when every row has the same scale."""
    g = np.random.default_rng(52)
    K = 64
    x = inputs.bf16_bits(g.standard_normal((3, K)).astype(np.float32))
    eye = _codes_of(np.eye(K), E5M2)
    s = (np.arange(1, K + 1) / 8.0).astype(np.float32)
    y, _ = oracle.weight_only_ref(x, eye, s, oracle.ROW, E5M2)
    assert np.array_equal(y, oracle.bf16_to_f32(x).astype(np.float64) * s.astype(np.float64)[None, :])
    w = g.integers(0, 256, (7, K)).astype(np.uint8)
    w[(w & 0x7F) == 0x7F] = 0          # keep E4M3 codes finite
    y1, _ = oracle.weight_only_ref(x, w, np.full(7, 0.25, np.float32), oracle.ROW, E4M3)
    y2, _ = oracle.weight_only_ref(x, w, np.array([0.25], np.float32), oracle.TENSOR, E4M3)
    assert np.array_equal(y1, y2)
