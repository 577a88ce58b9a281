"""GPU parity of fp8_quantize (through the C ABI) against the CPU oracle.

Codes, fp32 scales, E8M0 bytes and dequantised bf16 must be bit-exact: the
kernel and the oracle take every rounding decision in fp32 with the same
formula (s = fp32(max(amax, 1e-12f)/F_max), t = fp32(x/s), RNE cast)."""
import numpy as np
import pytest
import torch

import oracle
from fp8_dynamic_scaled_b200 import inputs
from gpu_util import first_mismatch, to_dev_bf16, to_host_u16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("fp8_dynamic_scaled_b200.binding") if torch.cuda.is_available() else None
if fp8 is None:
    pytest.skip("no CUDA device", allow_module_level=True)

FMTS = [fp8.FP8_E4M3, fp8.FP8_E5M2]
MODES = [fp8.FP8_SCALE_TENSOR, fp8.FP8_SCALE_ROW, fp8.FP8_SCALE_BLOCK_1x128, fp8.FP8_SCALE_BLOCK_128x128,
         fp8.FP8_SCALE_MX32]


def run_gpu(x_u16, fmt, mode, dequant=True, ld=None):
    rows, cols = x_u16.shape
    if ld is not None and ld != cols:
        buf = np.zeros((rows, ld), np.uint16)
        buf[:, :cols] = x_u16
        xd = to_dev_bf16(buf)[:, :cols]
    else:
        xd = to_dev_bf16(x_u16)
    q, s, d = fp8.empty_quant_outputs(rows, cols, mode, dequant=dequant)
    ws = fp8.workspace_for(0, rows, 0, cols, mode)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8.fp8_quantize(xd, fmt, mode, q, s, dequant=d, dev_status=st, workspace=ws)
    torch.cuda.synchronize()
    out = (q.cpu().numpy(), s.cpu().numpy(), to_host_u16(d) if d is not None else None, int(st.item()))
    return out


def check_parity(x_u16, fmt, mode, dequant=True, ld=None, what=""):
    q, s, d, st = run_gpu(x_u16, fmt, mode, dequant, ld)
    assert st == 0, f"{what}: dev_status {st}"
    rq, rs, rd = oracle.quantize(x_u16, fmt, mode, dequant=dequant)
    assert s.shape == rs.shape, (s.shape, rs.shape)
    mm = first_mismatch(s.view(np.uint32) if s.dtype == np.float32 else s,
                        rs.view(np.uint32) if rs.dtype == np.float32 else rs)
    assert mm is None, f"{what}: scale mismatch {mm}"
    mm = first_mismatch(q, rq)
    assert mm is None, f"{what}: code mismatch (index, gpu, oracle, count) {mm}"
    if dequant:
        mm = first_mismatch(d, rd)
        assert mm is None, f"{what}: dequant mismatch {mm}"


def mixed_input(rows, cols, seed):
    """Normal values times per-row lognormal magnitudes, with zeros, signed zeros,
    bf16 subnormals and a few large entries sprinkled in."""
    g = np.random.default_rng(seed)
    x = g.standard_normal((rows, cols)).astype(np.float32) * np.exp(2 * g.standard_normal((rows, 1))).astype(np.float32)
    n = rows * cols
    if n:
        flat = x.reshape(-1)
        k = max(1, n // 50)
        flat[g.integers(0, n, k)] = 0.0
        flat[g.integers(0, n, k)] = -0.0
        flat[g.integers(0, n, k)] = np.float32(3e-39) * g.choice([-1, 1], k)   # bf16 subnormals
        flat[g.integers(0, n, max(1, n // 997))] *= 1e4
    return inputs.bf16_bits(x)


SMALL_SHAPES = [(1, 16), (3, 48), (130, 256), (257, 384), (64, 1040), (129, 4096), (2, 2048 + 32)]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("shape", SMALL_SHAPES)
def test_quantize_small_shapes(fmt, mode, shape):
    rows, cols = shape
    if mode == fp8.FP8_SCALE_MX32 and (fmt != fp8.FP8_E4M3 or cols % 32):
        pytest.skip("MX32 is E4M3 with cols % 32 == 0")
    x = mixed_input(rows, cols, seed=rows * 7919 + cols)
    check_parity(x, fmt, mode, what=f"{shape} mode {mode} fmt {fmt}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("cols", [512, 2048])
def test_quantize_strided_rows(mode, cols):
    x = mixed_input(200, cols, seed=5)
    check_parity(x, fp8.FP8_E4M3, mode, ld=cols + 72, what=f"strided mode {mode}")


@pytest.mark.parametrize("mode", MODES)
def test_quantize_long_rows(mode):
    """Rows longer than one CTA holds in registers (second pass for ROW)."""
    x = mixed_input(3, 40960, seed=11)
    check_parity(x, fp8.FP8_E4M3, mode, what=f"long rows mode {mode}")


def test_quantize_all_zero_gives_floor_scale():
    x = np.zeros((64, 256), np.uint16)
    for mode in MODES:
        for fmt in FMTS:
            if mode == fp8.FP8_SCALE_MX32 and fmt != fp8.FP8_E4M3:
                continue
            check_parity(x, fmt, mode, what=f"zeros mode {mode}")


@pytest.mark.parametrize("mode", MODES)
def test_quantize_empty(mode):
    for rows, cols in ((0, 256), (5, 0), (0, 0)):
        q, s, d, st = run_gpu(np.zeros((rows, cols), np.uint16), fp8.FP8_E4M3, mode)
        rq, rs, rd = oracle.quantize(np.zeros((rows, cols), np.uint16), fp8.FP8_E4M3, mode)
        assert st == 0 and s.shape == rs.shape
        assert np.array_equal(s.view(np.uint32) if s.dtype == np.float32 else s,
                              rs.view(np.uint32) if rs.dtype == np.float32 else rs)


@pytest.mark.parametrize("cols", [256, 2048])
def test_quantize_nonfinite_sets_status(cols):
    for mode in MODES:
        x = mixed_input(32, cols, seed=3)
        x[5, 17] = 0x7F80   # +inf
        _, _, _, st = run_gpu(x, fp8.FP8_E4M3, mode)
        assert st == fp8.FP8_ERR_NONFINITE, (mode, st)
        x[5, 17] = 0xFFC1   # NaN
        _, _, _, st = run_gpu(x, fp8.FP8_E4M3, mode)
        assert st == fp8.FP8_ERR_NONFINITE, (mode, st)


def test_quantize_bad_arguments_rejected():
    x = torch.zeros((4, 24), dtype=torch.bfloat16, device="cuda")    # cols % 16 != 0
    q, s, _ = fp8.empty_quant_outputs(4, 24, fp8.FP8_SCALE_ROW)
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_quantize(x, fp8.FP8_E4M3, fp8.FP8_SCALE_ROW, q, s)
    assert e.value.status == fp8.FP8_ERR_INVALID_ARG
    x = torch.zeros((4, 32), dtype=torch.bfloat16, device="cuda")
    q, s, _ = fp8.empty_quant_outputs(4, 32, fp8.FP8_SCALE_TENSOR)
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_quantize(x, fp8.FP8_E4M3, fp8.FP8_SCALE_TENSOR, q, s, workspace=None)
    assert e.value.status == fp8.FP8_ERR_WORKSPACE
    q2, s2, _ = fp8.empty_quant_outputs(4, 32, fp8.FP8_SCALE_MX32)
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_quantize(x, fp8.FP8_E5M2, fp8.FP8_SCALE_MX32, q2, s2)
    assert e.value.status == fp8.FP8_ERR_INVALID_ARG


def _sweep_input(rows, cols, seed):
    """Rows whose elements are drawn from every finite bf16 magnitude below a random
    per-row amax (placed last in the row), with random signs."""
    g = np.random.default_rng(seed)
    pats = np.arange(0, 0x7F80, dtype=np.uint32)
    amax_pat = g.integers(0x3000, 0x7F7F, rows).astype(np.uint32)   # amax ~ 1e-10 .. 3e38
    x = np.zeros((rows, cols), np.uint16)
    for r in range(rows):
        below = pats[pats < amax_pat[r]]
        pick = g.choice(below, cols - 1, replace=below.size < cols - 1)
        sign = g.integers(0, 2, cols - 1).astype(np.uint32) << 15
        x[r, :cols - 1] = (pick | sign).astype(np.uint16)
        x[r, cols - 1] = amax_pat[r]
    return x


@pytest.mark.parametrize("mode", [fp8.FP8_SCALE_ROW, fp8.FP8_SCALE_BLOCK_1x128])
def test_cast_sweep_every_bf16_pattern_many_scales(mode):
    """Bf16 patterns of every magnitude under thousands of scales (one per row, or one
    per 1x128 block): about 67M (x, s) pairs per format through the division and the
    RNE cast, codes and dequant compared bit for bit."""
    x = _sweep_input(4096, 16384, seed=99 + mode)
    for fmt in FMTS:
        check_parity(x, fmt, mode, dequant=True, what=f"cast sweep mode {mode} fmt {fmt}")


def test_cast_sweep_long_rows_fallback():
    """Rows longer than the streaming kernel takes (second-pass row kernel)."""
    x = _sweep_input(512, 32640, seed=7)
    for fmt in FMTS:
        check_parity(x, fmt, fp8.FP8_SCALE_ROW, dequant=True, what=f"long-row sweep fmt {fmt}")


# ---------------------------------------------------------------- delayed scaling
def _dev_rows(x_u16, ld=None):
    """x on the device, with row stride ld (a view into a wider buffer) when given."""
    rows, cols = x_u16.shape
    if ld is None or ld == cols:
        return to_dev_bf16(x_u16)
    buf = np.zeros((rows, ld), np.uint16)
    buf[:, :cols] = x_u16
    return to_dev_bf16(buf)[:, :cols]


def run_delayed_sequence(xs, fmt, hist_len=16):
    hist = fp8.History(hist_len)
    ring = np.zeros(hist_len, np.float32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = None
    for t, x in enumerate(xs):
        rows, cols = x.shape
        if ws is None:
            ws = fp8.workspace_for(0, rows, 0, cols, fp8.FP8_SCALE_DELAYED)
        q, s, d = fp8.empty_quant_outputs(rows, cols, fp8.FP8_SCALE_DELAYED, dequant=True)
        fp8.fp8_quantize(to_dev_bf16(x), fmt, fp8.FP8_SCALE_DELAYED, q, s, hist=hist, dequant=d, dev_status=st,
                         workspace=ws)
        torch.cuda.synchronize()
        assert hist.step == t + 1
        rq, rs, rd, _ = oracle.delayed_step(x, fmt, ring, t, dequant=True)
        assert int(st.item()) == 0
        assert s.cpu().numpy().view(np.uint32)[0] == np.float32(rs).view(np.uint32), f"step {t} scale"
        mm = first_mismatch(q.cpu().numpy(), rq)
        assert mm is None, f"step {t} codes {mm}"
        assert first_mismatch(to_host_u16(d), rd) is None, f"step {t} dequant"
        assert np.array_equal(hist.ring.cpu().numpy().view(np.uint32), ring.view(np.uint32)), f"step {t} ring"
        assert hist.pending.item() == 0.0 and hist.ticket.item() == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_delayed_sixteen_steps_small(fmt):
    xs = [inputs.delayed_step_input(t, M=257, K=512) for t in range(20)]    # wraps the 16-entry ring
    run_delayed_sequence(xs, fmt)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("shape", [(256, 256), (64, 1024), (32, 2048 + 16), (1, 8192 * 8), (2, 8192 * 4 + 16)])
def test_per_tensor_around_the_single_cta_limit(fmt, shape):
    """Dense per-tensor tensors up to 65,536 elements take the one-CTA kernel, larger ones
    the two-pass kernels; both sides of the limit against the oracle."""
    check_parity(mixed_input(*shape, seed=sum(shape)), fmt, fp8.FP8_SCALE_TENSOR, what=f"per-tensor {shape}")


def test_delayed_small_tensor_single_cta():
    """Step 0 of a small delayed tensor runs in the one-CTA kernel and must record amax_0."""
    xs = [inputs.delayed_step_input(t, M=64, K=256) for t in range(6)]
    run_delayed_sequence(xs, fp8.FP8_E5M2, hist_len=4)


def test_delayed_short_history_and_strided_grid():
    xs = [mixed_input(1000, 1024, seed=t) for t in range(7)]
    run_delayed_sequence(xs, fp8.FP8_E4M3, hist_len=3)


# ---------------------------------------------------------------- full workload sizes
def test_quant_sweep_full_size_both_formats():
    """64 Mi-element log-uniform tensor with outliers, per-tensor, codes + scale + dequant."""
    x = inputs.quant_sweep()
    for fmt in FMTS:
        check_parity(x, fmt, fp8.FP8_SCALE_TENSOR, dequant=True, what=f"quant_sweep fmt {fmt}")


def test_llama70b_prefill_operands_full_size():
    x, w = inputs.llama70b_prefill()
    check_parity(x, fp8.FP8_E4M3, fp8.FP8_SCALE_ROW, dequant=False, what="X per-token")
    check_parity(w, fp8.FP8_E4M3, fp8.FP8_SCALE_ROW, dequant=False, what="W per-channel")


def test_block_scaled_operands_full_size():
    x, w = inputs.block_scaled()
    check_parity(x, fp8.FP8_E4M3, fp8.FP8_SCALE_BLOCK_1x128, dequant=False, what="X 1x128")
    check_parity(w, fp8.FP8_E4M3, fp8.FP8_SCALE_BLOCK_128x128, dequant=False, what="W 128x128")


def test_mx_operands_full_size():
    x, w = inputs.mx_delayed()
    check_parity(x, fp8.FP8_E4M3, fp8.FP8_SCALE_MX32, dequant=False, what="X MX32")
    check_parity(w, fp8.FP8_E4M3, fp8.FP8_SCALE_MX32, dequant=False, what="W MX32")


def test_delayed_full_size_sixteen_steps():
    """The whole drifting sequence at its full size: 16 steps of X_t [16384, 8192] with
    std 1 -> 4 and a 16-entry history; scale, codes, dequant and ring bit-exact every step."""
    base = inputs.delayed_base()
    xs = (inputs.delayed_step_input(t, base=base) for t in range(16))
    run_delayed_sequence(xs, fp8.FP8_E4M3)


# ---------------------------------------------------------------- non-finite delayed steps
@pytest.mark.parametrize("bad_step", [0, 5])
@pytest.mark.parametrize("bad", [0x7F80, 0xFFC1])          # +Inf, NaN
@pytest.mark.parametrize("shape,ld", [((64, 256), None),    # one-CTA step 0, then the dense single pass
                                      ((300, 1024), None),  # two-pass step 0, then the dense single pass
                                      ((200, 512), 584)])   # strided rows: the row-wise kernels
def test_delayed_nonfinite_step_records_nothing(bad_step, bad, shape, ld):
    """A delayed step whose input holds a NaN/Inf sets FP8_ERR_NONFINITE and leaves the
    history as it was; every later finite step is bit-exact with the oracle, which also
    refuses the bad step and records nothing ([FFS] "数值验证看什么": non-finite values
    are monitored, they must not reach the scale of the steps after them)."""
    rows, cols = shape
    h = 4
    hist = fp8.History(h)
    ring = np.zeros(h, np.float32)
    ws = fp8.workspace_for(0, rows, 0, cols, fp8.FP8_SCALE_DELAYED)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in range(9):
        x = mixed_input(rows, cols, seed=100 + t)
        if t == bad_step:
            x[rows // 2, cols // 3] = bad
        st.zero_()
        ring_before = hist.ring.cpu().numpy().copy()
        q, s, d = fp8.empty_quant_outputs(rows, cols, fp8.FP8_SCALE_DELAYED, dequant=True)
        fp8.fp8_quantize(_dev_rows(x, ld), fp8.FP8_E4M3, fp8.FP8_SCALE_DELAYED, q, s, hist=hist, dequant=d,
                         dev_status=st, workspace=ws)
        torch.cuda.synchronize()
        assert hist.step == t + 1
        assert hist.pending.item() == 0.0 and hist.ticket.item() == 0
        if t == bad_step:
            assert int(st.item()) == fp8.FP8_ERR_NONFINITE
            with pytest.raises(oracle.OracleError):
                oracle.delayed_step(x, fp8.FP8_E4M3, ring, t)
            assert np.array_equal(hist.ring.cpu().numpy().view(np.uint32), ring_before.view(np.uint32)), \
                "a non-finite step changed the history"
            assert np.array_equal(ring.view(np.uint32), ring_before.view(np.uint32))
            continue
        assert int(st.item()) == 0, f"step {t}"
        rq, rs, rd, _ = oracle.delayed_step(x, fp8.FP8_E4M3, ring, t, dequant=True)
        assert s.cpu().numpy().view(np.uint32)[0] == np.float32(rs).view(np.uint32), f"step {t} scale"
        assert first_mismatch(q.cpu().numpy(), rq) is None, f"step {t} codes"
        assert first_mismatch(to_host_u16(d), rd) is None, f"step {t} dequant"
        assert np.array_equal(hist.ring.cpu().numpy().view(np.uint32), ring.view(np.uint32)), f"step {t} ring"


def test_quantize_nonfinite_sets_status_delayed():
    """FP8_ERR_NONFINITE from the delayed mode at step 0 and at a later step."""
    for cols in (256, 2048):
        hist = fp8.History(16)
        for t in range(3):
            x = mixed_input(32, cols, seed=3 + t)
            x[5, 17] = 0x7F80 if t != 1 else 0xFFC1
            st = torch.zeros(1, dtype=torch.int32, device="cuda")
            q, s, d = fp8.empty_quant_outputs(32, cols, fp8.FP8_SCALE_DELAYED)
            fp8.fp8_quantize(to_dev_bf16(x), fp8.FP8_E4M3, fp8.FP8_SCALE_DELAYED, q, s, hist=hist, dev_status=st,
                             workspace=fp8.workspace_for(0, 32, 0, cols, fp8.FP8_SCALE_DELAYED))
            torch.cuda.synchronize()
            assert int(st.item()) == fp8.FP8_ERR_NONFINITE, (cols, t)
        assert np.all(hist.ring.cpu().numpy() == 0.0), "non-finite steps must record nothing"


# ---------------------------------------------------------------- MX32 extreme groups
def _mx_extreme_input(rows, cols, seed):
    """32-element groups whose amax spans the whole bf16 range: groups made only of bf16
    subnormals, normal groups below 2^-119 (the e = -127 clamp), groups just above it,
    and groups up to the largest finite bf16; elements are every magnitude at or below
    the group's amax (bf16 subnormals included), random signs."""
    g = np.random.default_rng(seed)
    ng = cols // 32
    amax = g.integers(0x0001, 0x7F80, (rows, ng)).astype(np.uint32)
    forced = np.array([0x0001, 0x0003, 0x003F, 0x0040, 0x007F, 0x0080, 0x0340, 0x0380, 0x03FF, 0x0400,
                       0x0480, 0x7F7F, 0x0000], np.uint32)
    amax[:, :min(ng, forced.size)] = forced[:min(ng, forced.size)]
    mags = (g.random((rows, ng, 32)) * (amax[:, :, None] + 1)).astype(np.uint32)
    # half of the elements at or below 2^-7 of the amax pattern's exponent: many subnormals
    small = g.random((rows, ng, 32)) < 0.5
    mags = np.where(small, mags & 0x00FF, mags)
    mags = np.minimum(mags, amax[:, :, None])
    pos = g.integers(0, 32, (rows, ng))
    np.put_along_axis(mags, pos[:, :, None], amax[:, :, None], axis=2)
    sign = g.integers(0, 2, (rows, ng, 32)).astype(np.uint32) << 15
    return (mags | sign).astype(np.uint16).reshape(rows, cols)


@pytest.mark.parametrize("shape,ld", [((64, 1024), None), ((130, 416), None), ((33, 2048), 2080),
                                      ((3, 40960), None)])
def test_mx_subnormal_and_clamped_groups(shape, ld):
    """MX32 groups at the bottom of the bf16 range: the subnormal-amax branch of the
    exponent and the clamp at e = -127 (byte 0x00), codes = encode(clip(x * 2^127));
    scale bytes, codes and dequant bit-exact with the oracle."""
    x = _mx_extreme_input(*shape, seed=shape[0] + shape[1])
    check_parity(x, fp8.FP8_E4M3, fp8.FP8_SCALE_MX32, dequant=True, ld=ld, what=f"mx extremes {shape}")
    _, e8, _ = oracle.quantize(x, oracle.E4M3, oracle.MX32, dequant=False)
    assert (e8 == 0).sum() > 0 and ((e8 > 0) & (e8 < 20)).sum() > 0


# ---------------------------------------------------------------- exhaustive cast sweep
_FINITE_MAGS = np.arange(0, 0x7F80, dtype=np.uint32)                     # every finite |bf16| pattern
_ALL_FINITE = np.concatenate([_FINITE_MAGS, _FINITE_MAGS | 0x8000]).astype(np.uint16)


def _sweep_amax_patterns():
    """>= 2,000 amax values: every 448 * 2^k and 57344 * 2^k that bf16 holds (power-of-two
    scales s = 2^j in both formats, since 57344 / 448 = 128, so x / s is exact and lands
    on every rounding midpoint of the FP8 grid, subnormal FP8 codes included), amax
    values whose scale is the 1e-12 floor, and random bf16 patterns."""
    pats = set()
    for base in (448.0, 57344.0):
        for k in range(-160, 130):
            v = np.ldexp(np.float64(base), k)
            if not (2.0 ** -133 <= v < 2.0 ** 128):
                continue
            b = int(inputs.bf16_bits(np.array([v], np.float32))[0])
            if 0 < b < 0x7F80 and float(inputs.bf16_to_f32(np.array([b], np.uint16))[0]) == v:
                pats.add(b)
    pats.update([0x0001, 0x0100, 0x2000, 0x2B8C, 0x7F7F])   # near the 1e-12 floor; the largest finite bf16
    g = np.random.default_rng(2024)
    pats.update(int(v) for v in g.integers(1, 0x7F80, 1900))
    return np.array(sorted(pats), np.uint32)


def _exhaustive_rows(amax_pats, cols=16384):
    """ROW sweep: for every amax A, rows holding A and every finite bf16 pattern (both
    signs) with |x| <= A, 16,383 per row (the last row of A padded by repetition)."""
    rows = []
    for a in amax_pats:
        p = _ALL_FINITE[(_ALL_FINITE & 0x7FFF) <= a]
        per = cols - 1
        nrow = -(-p.size // per)
        p = np.resize(p, nrow * per).reshape(nrow, per)
        rows.append(np.concatenate([p, np.full((nrow, 1), a, np.uint16)], axis=1))
    return np.concatenate(rows, axis=0)


def _exhaustive_blocks(amax_pats, cols=16384):
    """1x128 sweep: blocks of 127 patterns (every finite pattern with |x| <= A, both signs)
    plus A itself, for every amax A; blocks laid out 128 to a row."""
    blocks = []
    for a in amax_pats:
        p = _ALL_FINITE[(_ALL_FINITE & 0x7FFF) <= a]
        nb = -(-p.size // 127)
        p = np.resize(p, nb * 127).reshape(nb, 127)
        blocks.append(np.concatenate([np.full((nb, 1), a, np.uint16), p], axis=1))
    b = np.concatenate(blocks, axis=0)
    per_row = cols // 128
    nrow = -(-b.shape[0] // per_row)
    b = np.resize(b, (nrow * per_row, 128))
    return b.reshape(nrow, cols)


@pytest.mark.parametrize("mode", [fp8.FP8_SCALE_ROW, fp8.FP8_SCALE_BLOCK_1x128])
def test_cast_exhaustive_every_finite_bf16_pattern(mode):
    """Every finite bf16 pattern, both signs, through the cast under each of >= 2,000
    scales (one per row, or one per 1x128 block) and both formats, codes and dequant
    bit-exact with the oracle.  The power-of-two scales put x / s exactly on the FP8
    rounding midpoints (ties), where the kernel's reciprocal-plus-correction division
    must still equal the IEEE quotient ([FFS] "Scale 怎样把 Tensor 塞进 E4M3":
    X_fp8 = cast(clip(X / s)))."""
    amax = _sweep_amax_patterns()
    assert amax.size >= 2000
    x = _exhaustive_rows(amax) if mode == fp8.FP8_SCALE_ROW else _exhaustive_blocks(amax)
    for fmt in FMTS:
        check_parity(x, fmt, mode, dequant=True, what=f"exhaustive mode {mode} fmt {fmt}")


# ---------------------------------------------------------------- per-tensor in one launch
def _per_tensor_run(x_dev, fmt, ws, dequant=True):
    rows, cols = x_dev.shape
    q, s, d = fp8.empty_quant_outputs(rows, cols, fp8.FP8_SCALE_TENSOR, dequant=dequant)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8.fp8_quantize(x_dev, fmt, fp8.FP8_SCALE_TENSOR, q, s, dequant=d, dev_status=st, workspace=ws)
    torch.cuda.synchronize()
    return q, s, d, int(st.item())


def _check_against_oracle(x, q, s, d, fmt, what):
    rq, rs, rd = oracle.quantize(x, fmt, oracle.TENSOR, dequant=d is not None)
    assert s.cpu().numpy().view(np.uint32)[0] == rs.view(np.uint32)[0], f"{what}: scale"
    assert first_mismatch(q.cpu().numpy(), rq) is None, f"{what}: codes"
    if d is not None:
        assert first_mismatch(to_host_u16(d), rd) is None, f"{what}: dequant"


@pytest.mark.parametrize("shape", [(2048, 8192),      # 16 Mi elements: every CTA region fits on chip
                                   (2049, 8208),      # just above, ragged CTA regions
                                   (6000, 4096)])     # a spill part in every region
def test_per_tensor_single_launch_sizes(shape):
    """Dense per-tensor tensors from 16 Mi elements take the single-launch kernel (shared
    memory + registers + re-read spill, one grid-wide amax exchange); bit-exact with the
    oracle in both formats, codes + scale + dequant."""
    x = mixed_input(*shape, seed=shape[0])
    xd = to_dev_bf16(x)
    ws = fp8.workspace_for(0, shape[0], 0, shape[1], fp8.FP8_SCALE_TENSOR)
    for fmt in FMTS:
        q, s, d, st = _per_tensor_run(xd, fmt, ws)
        assert st == 0
        _check_against_oracle(x, q, s, d, fmt, f"single launch {shape} fmt {fmt}")


def test_per_tensor_single_launch_garbage_workspace_and_repeats():
    """The workspace needs no initialisation: filled with random bytes first, then reused
    by calls on changing inputs, the results stay bit-exact (each call's exchange only
    accepts slots tagged with its own call number)."""
    rows, cols = 4096, 4096
    n = fp8.fp8_workspace_size(0, rows, 0, cols, fp8.FP8_SCALE_TENSOR)
    ws = torch.randint(0, 256, (n,), dtype=torch.uint8, device="cuda")
    for i in range(4):
        x = mixed_input(rows, cols, seed=500 + i)
        if i == 2:
            x[17, 33] = 0x4F00            # a much larger amax than the calls before
        q, s, d, st = _per_tensor_run(to_dev_bf16(x), fp8.FP8_E4M3, ws)
        assert st == 0
        _check_against_oracle(x, q, s, d, fp8.FP8_E4M3, f"call {i}")


def test_per_tensor_single_launch_exchange_timeout_then_recovers():
    """A 1 ns limit makes the grid-wide exchange run out (every CTA but the last to arrive
    waits): FP8_ERR_TIMEOUT, no fault; after zeroing the workspace the same call at the
    default limit is bit-exact."""
    x = mixed_input(8192, 8192, seed=77)
    xd = to_dev_bf16(x)
    ws = fp8.workspace_for(0, 8192, 0, 8192, fp8.FP8_SCALE_TENSOR)
    seen = []
    fp8.fp8_testing_set_wait_limit_ns(1)
    try:
        for _ in range(3):
            seen.append(_per_tensor_run(xd, fp8.FP8_E4M3, ws)[3])
            if seen[-1] == fp8.FP8_ERR_TIMEOUT:
                break
    finally:
        fp8.fp8_testing_set_wait_limit_ns(0)
    assert fp8.FP8_ERR_TIMEOUT in seen, seen
    assert set(seen) <= {0, fp8.FP8_ERR_TIMEOUT}
    ws.zero_()
    q, s, d, st = _per_tensor_run(xd, fp8.FP8_E4M3, ws)
    assert st == 0
    _check_against_oracle(x, q, s, d, fp8.FP8_E4M3, "after the timeout")


def test_delayed_step0_single_launch_records_amax():
    """Step 0 of a large delayed history runs the single-launch kernel and records amax_0."""
    xs = [inputs.delayed_step_input(t, M=4096, K=8192) for t in range(3)]
    run_delayed_sequence(xs, fp8.FP8_E4M3, hist_len=4)
