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
def run_delayed_sequence(xs, fmt, hist_len=16):
    hist = fp8.History(hist_len)
    ring = np.zeros(hist_len, np.float32)
    ws = fp8.workspace_for(0, xs[0].shape[0], 0, xs[0].shape[1], fp8.FP8_SCALE_DELAYED)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t, x in enumerate(xs):
        rows, cols = x.shape
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


def test_delayed_full_size_first_steps():
    base = inputs.delayed_base()
    xs = [inputs.delayed_step_input(t, base=base) for t in range(3)]
    run_delayed_sequence(xs, fp8.FP8_E4M3)
