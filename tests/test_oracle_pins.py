"""Pins for the CPU oracle: each test checks the oracle against something other than
itself -- numbers printed on the pages (tests/golden), closed forms, invariants,
an independent brute-force search, and torch's CPU float8 casts (a library run
only as a third opinion).  Runs without a GPU."""
import numpy as np
import pytest
import torch

import oracle
from oracle import numpy_encoder
from conftest import read_golden
from fp8_dynamic_scaled_b200 import inputs

E4M3, E5M2 = oracle.E4M3, oracle.E5M2
TORCH_DT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


def torch_codes(v, fmt):
    return torch.from_numpy(np.asarray(v, np.float32)).to(TORCH_DT[fmt]).view(torch.uint8).numpy()


# ------------------------------------------------------------ format tables
def test_format_constants_match_pages():
    rows, _ = read_golden("format_constants.txt")
    for name, fmt in (("e4m3", E4M3), ("e5m2", E5M2)):
        sbits, ebits, mbits, bias, fmax = (float(t) for t in rows[name])
        assert oracle.fmax(fmt) == fmax
        # closed form (2 - 2^-2) * 2^emax with emax = 8 / 15
        emax = 8 if fmt == E4M3 else 15
        assert oracle.fmax(fmt) == (2 - 2 ** -2) * 2 ** emax
        # the bias: code with exponent field == bias and zero mantissa is 1.0
        one = int(bias) << int(mbits)
        assert oracle.decode(one, fmt) == 1.0
        # min normal 2^(1-bias), min subnormal 2^(1-bias-mbits)
        assert oracle.decode(1 << int(mbits), fmt) == 2.0 ** (1 - bias)
        assert oracle.decode(1, fmt) == 2.0 ** (1 - bias - mbits)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_code_table_counts_and_monotone(fmt):
    t = oracle.decode_table(fmt)
    n_nan = int(np.isnan(t).sum())
    n_inf = int(np.isinf(t).sum())
    n_fin = int(np.isfinite(t).sum())
    if fmt == E4M3:
        assert (n_fin, n_nan, n_inf) == (254, 2, 0)
        assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    else:
        assert (n_fin, n_nan, n_inf) == (248, 6, 2)
        assert t[0x7C] == np.inf and t[0xFC] == -np.inf
    pos = t[:128][np.isfinite(t[:128])]
    assert np.all(np.diff(pos) > 0), "positive finite codes must be strictly increasing"
    neg = t[128:][np.isfinite(t[128:])]
    assert np.array_equal(neg, -pos)
    assert t[0] == 0.0 and t[0x80] == 0.0 and np.signbit(t[0x80])


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_decode_table_matches_independent_table_and_torch(fmt):
    t = oracle.decode_table(fmt)
    u = numpy_encoder.value_table(fmt)
    both_nan = np.isnan(t) & np.isnan(u)
    assert np.all(both_nan | (t == u))
    tt = torch.arange(256, dtype=torch.uint8).view(TORCH_DT[fmt]).to(torch.float64).numpy()
    assert np.all((np.isnan(t) & np.isnan(tt)) | (t == tt))


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_roundtrip_every_finite_code(fmt):
    t = oracle.decode_table(fmt)
    codes = np.nonzero(np.isfinite(t))[0]
    enc = oracle.encode(t[codes].astype(np.float32), fmt)
    assert np.array_equal(enc, codes.astype(np.uint8))


# ------------------------------------------------------------ encoder pins
def _midpoints(fmt):
    t = oracle.decode_table(fmt)
    pos = t[:128][np.isfinite(t[:128])]
    mids = (pos[:-1] + pos[1:]) / 2.0
    m32 = mids.astype(np.float32)
    assert np.all(m32.astype(np.float64) == mids)       # midpoints are exact in fp32
    up = np.nextafter(m32, np.float32(np.inf))
    dn = np.nextafter(m32, np.float32(0))
    v = np.concatenate([m32, up, dn, pos.astype(np.float32)])
    return np.concatenate([v, -v])


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encoder_midpoints_against_bruteforce_numpy_and_torch(fmt):
    v = _midpoints(fmt)
    a = oracle.encode(v, fmt)
    assert np.array_equal(a, oracle.encode_bruteforce(v, fmt))
    assert np.array_equal(a, numpy_encoder.encode_nearest(v, fmt))
    assert np.array_equal(a, torch_codes(v, fmt))


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encoder_random_against_bruteforce_and_torch(fmt):
    F = oracle.fmax(fmt)
    g = np.random.default_rng(7)
    n = 1_000_000
    lo = -12 if fmt == E4M3 else -19
    mag = np.exp2(g.uniform(lo, np.log2(F), size=n))
    v = (mag * np.where(g.integers(0, 2, n) == 1, -1, 1)).astype(np.float32)
    v = np.clip(v, -F, F).astype(np.float32)
    a = oracle.encode(v, fmt)
    assert np.array_equal(a, oracle.encode_bruteforce(v, fmt))
    assert np.array_equal(a, torch_codes(v, fmt))
    sub = v[:20000]
    assert np.array_equal(a[:20000], numpy_encoder.encode_nearest(sub, fmt))


def test_signed_zero_and_tiny_negatives():
    for fmt in (E4M3, E5M2):
        tiny = 2.0 ** (-11 if fmt == E4M3 else -18)
        v = np.array([0.0, -0.0, -tiny, tiny], np.float32)
        assert list(oracle.encode(v, fmt)) == [0x00, 0x80, 0x80, 0x00]


# ------------------------------------------------------------ page examples
@pytest.mark.parametrize("fmt,col", [(E4M3, 2), (E5M2, 3)])
def test_fpi_dequant_worked_example(fmt, col):
    rows, table = read_golden("fpi_dequant_example.txt")
    s = np.float32(float(rows["scale"][0]))
    vals = np.array([float(r[0]) for r in table], np.float32)
    printed = np.array([float(r[1]) for r in table])
    codes = oracle.encode(vals, fmt)
    assert list(codes) == [int(r[col], 16) for r in table]
    dec = np.array([oracle.decode(int(c), fmt) for c in codes], np.float32)
    deq = dec * s                                  # fp32 product, as the path computes it
    ulp = np.spacing(np.abs(printed).astype(np.float32))
    assert np.all(np.abs(deq.astype(np.float64) - printed) <= ulp)


@pytest.mark.parametrize("fmt,col", [(E4M3, 2), (E5M2, 3)])
def test_dequant_scaled_worked_example(fmt, col):
    """[FPI] "反量化示例" through the oracle's dequantiser: bf16 of fp32(decode(q) * 0.01)
    lies within one bf16 step of the printed 0.0125, -0.005, 0.03."""
    rows, table = read_golden("fpi_dequant_example.txt")
    codes = np.array([int(r[col], 16) for r in table], np.uint8)
    printed = np.array([float(r[1]) for r in table])
    got = oracle.bf16_to_f32(oracle.dequant_scaled(codes, float(rows["scale"][0]), fmt)).astype(np.float64)
    step = np.array([oracle.bf16_ulp(v) for v in printed])
    assert np.all(np.abs(got - printed) <= step)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_dequant_scaled_exact_cases_and_torch(fmt):
    """Every FP8 value is a bf16 value, so a unit or power-of-two scale dequantises
    exactly; NaN codes stay NaN and E5M2's infinities stay infinite; any other scale
    gives the bf16 rounding of the fp32 product, as torch computes it."""
    codes = np.arange(256, dtype=np.uint8)
    table = oracle.decode_table(fmt)
    fin = np.isfinite(table)
    for k in (0, -7, 5, -20):
        got = oracle.bf16_to_f32(oracle.dequant_scaled(codes, 2.0 ** k, fmt)).astype(np.float64)
        assert np.array_equal(got[fin], table[fin] * 2.0 ** k)
        assert np.all(np.isnan(got[np.isnan(table)]))
        assert np.array_equal(got[np.isinf(table)], table[np.isinf(table)])
    g = np.random.default_rng(71 + fmt)
    for s in np.float32(10.0) ** g.uniform(-8, 3, 6).astype(np.float32):
        got = oracle.dequant_scaled(codes[fin], float(s), fmt)
        ref = (torch.from_numpy(table[fin].astype(np.float32)) * torch.tensor(float(s), dtype=torch.float32))
        assert np.array_equal(got, ref.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


def test_ffs_outlier_example():
    rows, table = read_golden("ffs_outlier_example.txt")
    x = np.array([float(r[0]) for r in table], np.float32)
    s = oracle.scale_from_amax(float(rows["outlier"][0]), E4M3)
    assert s == np.float32(np.float32(400.0) / np.float32(448.0))
    assert abs(s - float(rows["scale_num"][0]) / float(rows["scale_den"][0])) < 1e-7
    codes = oracle.quant_scaled(x, s, E4M3)
    assert list(codes) == [int(r[1], 16) for r in table]
    assert [oracle.decode(int(c), E4M3) for c in codes] == [float(r[2]) for r in table]
    # the same numbers through the full per-tensor quantize of a bf16 matrix
    xb = inputs.bf16_bits(x.reshape(1, -1))
    q, sc, _ = oracle.quantize(xb, E4M3, oracle.TENSOR, dequant=False)
    assert sc[0] == s and list(q[0]) == list(codes)


def test_frlp_vector_current_scaling():
    _, table = read_golden("frlp_test_vector.txt")
    x = np.array([[float(r[0]) for r in table]], np.float32)
    q, s, _ = oracle.quantize(inputs.bf16_bits(x), E4M3, oracle.TENSOR, dequant=False)
    assert np.isfinite(s[0]) and s[0] > 0
    assert s[0] == np.float32(np.float32(3.0) / np.float32(448.0))
    assert list(q[0]) == [int(r[1], 16) for r in table]


# ------------------------------------------------------------ scale invariants
@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_zero_input_gives_finite_positive_scale(fmt):
    z = np.zeros((3, 64), np.uint16)
    for mode in (oracle.TENSOR, oracle.ROW, oracle.BLOCK_1x128, oracle.BLOCK_128x128):
        q, s, d = oracle.quantize(z, fmt, mode)
        assert np.all(np.isfinite(s)) and np.all(s > 0)
        assert np.all(s == np.float32(np.float32(1e-12) / np.float32(oracle.fmax(fmt))))
        assert not q.any() and not d.any()
    if fmt == E4M3:
        q, s, d = oracle.quantize(z, fmt, oracle.MX32)
        assert np.all(s == 0) and not q.any()


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_amax_maps_to_fmax(fmt):
    g = np.random.default_rng(3)
    x = inputs.bf16_bits(g.standard_normal((64, 256)).astype(np.float32) * 3)
    xf = inputs.bf16_to_f32(x)
    top = 0x7E if fmt == E4M3 else 0x7B
    for mode in (oracle.TENSOR, oracle.ROW, oracle.BLOCK_1x128):
        q, s, _ = oracle.quantize(x, fmt, mode, dequant=False)
        if mode == oracle.TENSOR:
            groups = [np.ones_like(xf, bool)]
        elif mode == oracle.ROW:
            groups = [np.arange(64)[:, None] == r for r in range(64)]
            groups = [np.broadcast_to(gm, xf.shape) for gm in groups]
        else:
            groups = []
            for r in range(64):
                for b in range(2):
                    gm = np.zeros_like(xf, bool)
                    gm[r, b * 128:(b + 1) * 128] = True
                    groups.append(gm)
        for gm in groups:
            a = np.abs(xf[gm]).max()
            hits = q[gm & (np.abs(xf) == a)]
            assert np.all((hits & 0x7F) == top)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_dequant_error_within_half_quantum(fmt):
    """Unsaturated elements: |s*decode(q) - x| <= 1/2 quantum(q)*s (plus fp32 rounding)."""
    g = np.random.default_rng(11)
    x = inputs.bf16_bits(g.standard_normal((32, 512)).astype(np.float32))
    xf = inputs.bf16_to_f32(x).astype(np.float64)
    q, s, d = oracle.quantize(x, fmt, oracle.ROW)
    dec = oracle.decode_table(fmt)[q]
    mbits = 3 if fmt == E4M3 else 2
    emin = -6 if fmt == E4M3 else -14
    a = np.abs(xf / s[:, None])
    e = np.maximum(np.floor(np.log2(np.maximum(a, 2.0 ** emin))), emin)
    quantum = np.exp2(e - mbits)
    err = np.abs(dec * s[:, None] - xf)
    assert np.all(err <= 0.5 * quantum * s[:, None] * (1 + 1e-6) + 1e-30)
    # dequant output is the bf16 rounding of fp32(decode * s)
    want = oracle.f32_to_bf16((dec.astype(np.float32) * s[:, None].astype(np.float32)))
    assert np.array_equal(d, want)


def test_quantization_is_monotone():
    v = np.sort(np.random.default_rng(5).uniform(-3, 3, 4096).astype(np.float32))
    for fmt in (E4M3, E5M2):
        q = oracle.quant_scaled(v, 3.0 / oracle.fmax(fmt), fmt)
        dec = oracle.decode_table(fmt)[q]
        assert np.all(np.diff(dec) >= 0)


def test_bf16_rounding_matches_torch():
    g = np.random.default_rng(9)
    v = np.concatenate([g.standard_normal(100000).astype(np.float32) * 1e3,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8], np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16(v), ref)
    assert np.array_equal(inputs.bf16_bits(v), ref)


# ------------------------------------------------------------ block and MX modes
def test_block_modes_scale_layout():
    """Per-block scale = amax of exactly that block / F (checked with numpy reshapes)."""
    g = np.random.default_rng(13)
    rows, cols = 200, 384          # ragged in rows for 128x128
    x = inputs.bf16_bits(g.standard_normal((rows, cols)).astype(np.float32)
                         * np.exp(g.standard_normal((rows, 1))).astype(np.float32))
    xf = np.abs(inputs.bf16_to_f32(x))
    F = np.float32(448.0)
    _, s1, _ = oracle.quantize(x, E4M3, oracle.BLOCK_1x128, dequant=False)
    a1 = xf.reshape(rows, 3, 128).max(axis=2)
    assert np.array_equal(s1, np.maximum(a1, np.float32(1e-12)) / F)
    _, s2, _ = oracle.quantize(x, E4M3, oracle.BLOCK_128x128, dequant=False)
    pad = np.zeros((256, cols), np.float32)
    pad[:rows] = xf
    a2 = pad.reshape(2, 128, 3, 128).max(axis=(1, 3))
    assert np.array_equal(s2, np.maximum(a2, np.float32(1e-12)) / F)


def test_mx32_exponent_range_and_codes():
    g = np.random.default_rng(17)
    x = inputs.bf16_bits((g.standard_normal((16, 256))
                          * np.exp2(g.integers(-20, 20, (16, 1)))).astype(np.float32))
    xf = inputs.bf16_to_f32(x)
    q, e8, _ = oracle.quantize(x, E4M3, oracle.MX32, dequant=False)
    amax = np.abs(xf).reshape(16, 8, 32).max(axis=2)
    e = e8.astype(np.int64) - 127
    r = amax / np.exp2(e)
    assert np.all((r >= 256) & (r < 512))
    # codes equal the encoding of clip(x * 2^-e) (a power-of-two scale is exact)
    t = np.clip(xf.reshape(16, 8, 32) * np.exp2(-e)[:, :, None], -448, 448)
    assert np.array_equal(q, oracle.encode(t.astype(np.float32), E4M3).reshape(16, 256))
    assert oracle.mx_exponent(0.0) == -127


def _frexp_floor_log2(v: float) -> int:
    """floor(log2 v) of a positive float through Python's own frexp (independent of the oracle)."""
    import math
    return math.frexp(v)[1] - 1


def test_mx32_subnormal_and_clamped_groups():
    """Groups whose amax is a bf16 subnormal, or a normal below 2^-119, reach the lower
    clamp e = -127 ([FFS] "Per-channel 与 Block Scaling": one power-of-two scale per 32
    values; e = clamp(floor(log2 amax) - 8, -127, 127)): the scale byte is 0x00 and the
    codes are the nearest-code encoding of clip(x * 2^127), which the NumPy brute-force
    encoder computes here independently.  Groups just above the clamp keep e exact."""
    from oracle import numpy_encoder
    # amax patterns: bf16 subnormals 2^-133, 3*2^-132, 2^-127 (0x0040), and normals
    # 1.5*2^-121, 2^-120, 2^-119 (e = -127 exactly), 2^-118 (e = -126), 1.75*2^-101
    amax_bits = np.array([0x0001, 0x0003, 0x0040, 0x0340, 0x0380, 0x0400, 0x0480, 0x0D60], np.uint16)
    g = np.random.default_rng(23)
    x = np.zeros((4, 32 * amax_bits.size), np.uint16)
    for j, a in enumerate(amax_bits):
        # every element of the group at or below its amax pattern, random signs; the
        # amax itself at a random position
        mags = g.integers(0, int(a) + 1, (4, 32)).astype(np.uint16)
        mags[np.arange(4), g.integers(0, 32, 4)] = a
        sign = (g.integers(0, 2, (4, 32)) << 15).astype(np.uint16)
        x[:, 32 * j:32 * (j + 1)] = mags | sign
    q, e8, d = oracle.quantize(x, E4M3, oracle.MX32, dequant=True)
    amax_f = inputs.bf16_to_f32(amax_bits).astype(np.float64)
    e_expect = np.array([min(127, max(-127, _frexp_floor_log2(v) - 8)) for v in amax_f])
    assert e_expect[:6].tolist() == [-127] * 6 and e_expect[6] == -126 and e_expect[7] == -109
    assert np.array_equal(e8.astype(np.int64) - 127, np.tile(e_expect, (4, 1)))
    assert np.all(e8[:, :6] == 0)
    xf = inputs.bf16_to_f32(x).astype(np.float64)
    t = np.clip(xf * np.exp2(-np.repeat(e_expect, 32))[None, :], -448.0, 448.0)
    ref = numpy_encoder.encode_nearest(t.ravel(), E4M3).reshape(q.shape)
    assert np.array_equal(q, ref)
    # dequant: decode(q) * 2^e, exact in fp32, then bf16 (here every value is a bf16 value
    # or a bf16 subnormal rounding case handled by the torch cast)
    import torch
    table = numpy_encoder.value_table(E4M3)
    dq = (table[q] * np.exp2(np.repeat(e_expect, 32))[None, :]).astype(np.float32)
    dt = torch.from_numpy(dq).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(d, dt)


# ------------------------------------------------------------ delayed scaling
def test_delayed_nonfinite_step_records_nothing():
    """A step whose input holds a NaN or an Inf is refused and leaves the history as it
    was; the steps after it take their scale from the window of the valid steps only
    (written out here as a plain list of the amax of each valid step)."""
    g = np.random.default_rng(29)
    h = 4
    ring = np.zeros(h, np.float32)
    slot_amax = {}                      # slot -> amax of the last valid step that wrote it
    for t in range(11):
        x = inputs.bf16_bits((g.standard_normal((8, 64)) * (1 + t)).astype(np.float32))
        if t in (2, 7):
            x[3, 5] = 0x7F80 if t == 2 else 0xFFC1        # +Inf, NaN
            before = ring.copy()
            with pytest.raises(oracle.OracleError):
                oracle.delayed_step(x, E4M3, ring, t)
            assert np.array_equal(ring.view(np.uint32), before.view(np.uint32))
            continue
        xf = inputs.bf16_to_f32(x)
        amax_t = np.float32(np.abs(xf).max())
        q, s, _, _ = oracle.delayed_step(x, E4M3, ring, t)
        if t == 0:
            hist = amax_t
        else:
            hist = np.float32(max(slot_amax.values(), default=np.float32(0)))
        assert s == np.float32(max(hist, np.float32(1e-12)) / np.float32(448.0)), t
        assert np.array_equal(q, oracle.quant_scaled(xf.ravel(), s, E4M3).reshape(q.shape))
        slot_amax[t % h] = amax_t
    # slot 2 % 4 = 2 was last written by step 10; slot 7 % 4 = 3 by step 3 (step 7 was refused)
    assert ring[3] == slot_amax[3]


def test_delayed_ring_semantics():
    g = np.random.default_rng(19)
    h = 4
    ring = np.zeros(h, np.float32)
    amaxes = []
    for t in range(10):
        x = inputs.bf16_bits((g.standard_normal((8, 64)) * (1 + t)).astype(np.float32))
        xf = inputs.bf16_to_f32(x)
        amax_t = np.float32(np.abs(xf).max())
        q, s, _, sat = oracle.delayed_step(x, E4M3, ring, t)
        if t == 0:
            hist = amax_t
        else:
            hist = np.float32(max(amaxes[max(0, t - h):t]))    # window of the last h steps
        assert s == np.float32(max(hist, np.float32(1e-12)) / np.float32(448.0))
        assert sat == int((np.abs(xf / s) > 448).sum())
        ref_q = oracle.quant_scaled(xf.ravel(), s, E4M3).reshape(q.shape)
        assert np.array_equal(q, ref_q)
        amaxes.append(amax_t)
        assert ring[t % h] == amax_t
    assert sorted(ring.tolist()) == sorted(amaxes[-h:])


def test_delayed_drift_saturates():
    """Growing std with a stale window max saturates some elements (the risk the
    'Delayed Scaling' section names)."""
    ring = np.zeros(16, np.float32)
    sats = []
    for t in range(4):
        x = inputs.delayed_step_input(t, M=64, K=256)
        _, _, _, sat = oracle.delayed_step(x, E4M3, ring, t)
        sats.append(sat)
    assert sats[0] == 0 and max(sats[1:]) > 0


# ------------------------------------------------------------ GEMM reference
def _codes_of(values, fmt):
    return oracle.encode(np.asarray(values, np.float32), fmt).reshape(np.shape(values))


def test_gemm_ref_exact_integer_case():
    """Small-integer codes, unit scales: the reference equals an int64 matmul."""
    g = np.random.default_rng(23)
    M, N, K = 7, 5, 96
    a_int = g.integers(-8, 9, (M, K))
    b_int = g.integers(-8, 9, (N, K))
    a = _codes_of(a_int, E4M3)
    b = _codes_of(b_int, E5M2)
    one = np.ones(1, np.float32)
    y, bound = oracle.gemm_ref_full(a, one, oracle.TENSOR, E4M3, b, one, oracle.TENSOR, E5M2)
    assert np.array_equal(y, (a_int @ b_int.T).astype(np.float64))
    assert np.array_equal(bound, (np.abs(a_int) @ np.abs(b_int).T).astype(np.float64))


def test_gemm_ref_scales_expanded_independently():
    """Row/block/MX scales applied by explicit expansion + numpy matmul agree with the oracle."""
    g = np.random.default_rng(29)
    M, N, K = 130, 136, 256
    x = inputs.bf16_bits((g.standard_normal((M, K)) * np.exp(g.standard_normal((M, 1)))).astype(np.float32))
    w = inputs.bf16_bits((g.standard_normal((N, K)) * 0.02).astype(np.float32))
    dec4 = numpy_encoder.value_table(E4M3)
    cases = [(oracle.ROW, oracle.ROW), (oracle.BLOCK_1x128, oracle.BLOCK_128x128),
             (oracle.MX32, oracle.MX32), (oracle.TENSOR, oracle.ROW)]
    for am, bm in cases:
        qa, sa, _ = oracle.quantize(x, E4M3, am, dequant=False)
        qb, sb, _ = oracle.quantize(w, E4M3, bm, dequant=False)

        def expand(s, mode, rows):
            if mode == oracle.TENSOR:
                return np.full((rows, K), s[0], np.float64)
            if mode == oracle.ROW:
                return np.repeat(s[:, None].astype(np.float64), K, axis=1)
            if mode == oracle.BLOCK_1x128:
                return np.repeat(s.astype(np.float64), 128, axis=1)[:, :K]
            if mode == oracle.BLOCK_128x128:
                return np.repeat(np.repeat(s.astype(np.float64), 128, axis=0), 128, axis=1)[:rows, :K]
            return np.repeat(np.exp2(s.astype(np.float64) - 127), 32, axis=1)

        da = dec4[qa] * expand(sa, am, M)
        db = dec4[qb] * expand(sb, bm, N)
        y, bound = oracle.gemm_ref_full(qa, sa, am, E4M3, qb, sb, bm, E4M3)
        assert np.all(np.abs(y - da @ db.T) <= 1e-12 * (np.abs(da) @ np.abs(db).T))
        assert np.allclose(bound, np.abs(da) @ np.abs(db).T, rtol=1e-12)
        pm = g.integers(0, M, 50)
        pn = g.integers(0, N, 50)
        yp, bp = oracle.gemm_ref_points(qa, sa, am, E4M3, qb, sb, bm, E4M3, pm, pn)
        assert np.array_equal(yp, y[pm, pn]) and np.array_equal(bp, bound[pm, pn])


def test_gemm_identity_weight():
    """W = I (per-tensor, s_w from amax 1): Y = s_x * s_w * decode(q_x)."""
    K = 64
    g = np.random.default_rng(31)
    x = inputs.bf16_bits(g.standard_normal((9, K)).astype(np.float32))
    w = inputs.bf16_bits(np.eye(K, dtype=np.float32))
    qa, sa, _ = oracle.quantize(x, E4M3, oracle.TENSOR, dequant=False)
    qb, sb, _ = oracle.quantize(w, E4M3, oracle.TENSOR, dequant=False)
    assert sb[0] == np.float32(1.0 / 448.0) and np.all(qb[np.eye(K, dtype=bool)] == 0x7E)
    y, _ = oracle.gemm_ref_full(qa, sa, oracle.TENSOR, E4M3, qb, sb, oracle.TENSOR, E4M3)
    want = numpy_encoder.value_table(E4M3)[qa] * float(sa[0]) * 448.0 * float(sb[0])
    assert np.allclose(y, want, rtol=1e-15, atol=0)


def test_tolerance_rule_rejects_planted_error():
    y = np.array([1.0, 100.0, -3.0])
    bound = np.array([10.0, 200.0, 3.0])
    ok, _, _ = oracle.gemm_within_tolerance(y, y, bound)
    assert ok.all()
    bad = y + 1e-3 * bound + 4 * oracle.bf16_ulp(y)
    ok, _, _ = oracle.gemm_within_tolerance(bad, y, bound)
    assert not ok.any()
    assert oracle.bf16_ulp(np.array([1.0]))[0] == 2 ** -7


def test_results_do_not_depend_on_the_thread_count():
    """The oracle splits rows (and output points) over threads; every mode gives the same
    bits on 1 thread and on several, including the ragged last range."""
    x = inputs.bf16_bits((np.random.default_rng(31).standard_normal((259, 512))
                          * np.exp(np.random.default_rng(32).standard_normal((259, 1)))).astype(np.float32))
    w = inputs.bf16_bits((np.random.default_rng(33).standard_normal((140, 512)) * 0.02).astype(np.float32))
    prev = oracle.get_threads()
    try:
        outs = {}
        for n in (1, 5):
            oracle.set_threads(n)
            res = [oracle.quantize(x, fmt, mode) for fmt in (E4M3, E5M2) for mode in
                   (oracle.TENSOR, oracle.ROW, oracle.BLOCK_1x128, oracle.BLOCK_128x128)]
            res.append(oracle.quantize(x, E4M3, oracle.MX32))
            ring = np.zeros(4, np.float32)
            res.append(tuple(oracle.delayed_step(x, E4M3, ring, t)[:2] for t in range(3)) + (ring.copy(),))
            qa, sa, _ = oracle.quantize(x, E4M3, oracle.ROW, dequant=False)
            qb, sb, _ = oracle.quantize(w, E4M3, oracle.ROW, dequant=False)
            pm = np.repeat(np.arange(259), 7)
            pn = np.tile(np.arange(0, 140, 20), 259)
            res.append(oracle.gemm_ref_points(qa, sa, oracle.ROW, E4M3, qb, sb, oracle.ROW, E4M3, pm, pn))
            v = np.arange(0x3B000000, 0x3B000000 + 100003, dtype=np.uint32).view(np.float32)   # ragged ranges
            res.extend(oracle.encode(v, fmt) for fmt in (E4M3, E5M2))
            res.extend(oracle.quant_scaled(v, 0.75, fmt) for fmt in (E4M3, E5M2))
            outs[n] = res
        def flat(r):
            out = []
            for v in r:
                if isinstance(v, (tuple, list)):
                    out.extend(flat(v))
                elif v is not None:
                    out.append(np.atleast_1d(np.asarray(v)))
            return out
        a, b = flat(outs[1]), flat(outs[5])
        assert len(a) == len(b)
        for u, v in zip(a, b):
            assert np.array_equal(u.view(np.uint8) if u.dtype.kind == "f" else u,
                                  v.view(np.uint8) if v.dtype.kind == "f" else v)
    finally:
        oracle.set_threads(prev)


def test_gemm_ref_rows_agrees_with_the_pointwise_reference():
    """gemm_ref_rows (fp64 BLAS over exactly dequantised operands) against the C
    reference at every output of small problems in every scale mode, to fp64 rounding."""
    g = np.random.default_rng(37)
    cases = [(oracle.ROW, oracle.ROW, E4M3, E5M2), (oracle.TENSOR, oracle.TENSOR, E5M2, E5M2),
             (oracle.BLOCK_1x128, oracle.BLOCK_128x128, E4M3, E4M3), (oracle.MX32, oracle.MX32, E4M3, E4M3)]
    for am, bm, fa, fb in cases:
        M, N, K = 130, 260, 384
        x = inputs.bf16_bits((g.standard_normal((M, K)) * np.exp(g.standard_normal((M, 1)))).astype(np.float32))
        w = inputs.bf16_bits((g.standard_normal((N, K)) * 0.02).astype(np.float32))
        qa, sa, _ = oracle.quantize(x, fa, am, dequant=False)
        qb, sb, _ = oracle.quantize(w, fb, bm, dequant=False)
        y, bnd = oracle.gemm_ref_full(qa, sa, am, fa, qb, sb, bm, fb)
        rows = np.array([0, 1, 64, 127, 128, 129])
        y2, b2 = oracle.gemm_ref_rows(qa, sa, am, fa, qb, sb, bm, fb, rows, chunk=100)
        assert np.allclose(y2, y[rows], rtol=0, atol=1e-12 * bnd[rows].max())
        assert np.allclose(b2, bnd[rows], rtol=1e-12, atol=0)
