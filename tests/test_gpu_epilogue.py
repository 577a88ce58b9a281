"""GPU parity of the split per-tensor scaling (fp8_amax, fp8_quantize_with_amax) and of
the GEMM epilogue options (bias, output amax, FP8 output codes) through the C ABI.

References: the oracle's amax and given-amax cast (bit-exact); for the GEMM, the
oracle's fp64 result plus bias under the usual acceptance rule, the interval of
admissible FP8 output codes that the rule implies (the quantiser is monotone), and
bit-exact results where the arithmetic is exact (small integers, unit scales).
Where a result is defined through another output of the same call (the output
amax is the maximum of the stored Y), the two GPU outputs are compared with each
other."""
import numpy as np
import pytest
import torch

import oracle
from fp8_dynamic_scaled_b200 import inputs
from gpu_util import assert_gemm_close, bf16_bits_to_f64, first_mismatch, to_dev_bf16, to_host_u16

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
import fp8_dynamic_scaled_b200.binding as fp8  # noqa: E402

E4M3, E5M2 = fp8.FP8_E4M3, fp8.FP8_E5M2
T, R, B1, B128, MX = (fp8.FP8_SCALE_TENSOR, fp8.FP8_SCALE_ROW, fp8.FP8_SCALE_BLOCK_1x128,
                      fp8.FP8_SCALE_BLOCK_128x128, fp8.FP8_SCALE_MX32)


def dev_f32(v):
    return torch.tensor(np.atleast_1d(np.asarray(v, np.float32)), device="cuda")


def status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def rand_bf16(shape, seed, std=1.0, spread=0.0):
    g = np.random.default_rng(seed)
    x = g.standard_normal(shape).astype(np.float32) * np.float32(std)
    if spread:
        x *= np.exp(g.standard_normal((shape[0], 1)) * spread).astype(np.float32)
    return inputs.bf16_bits(x)


# ================================================================ fp8_amax
def gpu_amax(x_dev):
    rows, cols = x_dev.shape
    a = dev_f32(-1.0)
    st = status()
    ws = fp8.workspace_for(0, rows, 0, cols, T)
    fp8.fp8_amax(x_dev, a, dev_status=st, workspace=ws)
    torch.cuda.synchronize()
    return float(a.item()), int(st.item())


@pytest.mark.parametrize("rows,cols", [(1, 16), (7, 48), (128, 256), (333, 1040), (4096, 8192)])
def test_amax_matches_oracle(rows, cols):
    x = rand_bf16((rows, cols), seed=rows + cols, spread=3.0)
    a, st = gpu_amax(to_dev_bf16(x))
    assert st == 0 and a == oracle.amax(x)


def test_amax_strided_zero_empty_and_nonfinite():
    x = rand_bf16((65, 512), seed=3, spread=2.0)
    big = to_dev_bf16(x)
    view = big[:, 64:64 + 256]
    a, st = gpu_amax(view)
    assert st == 0 and a == oracle.amax(x[:, 64:64 + 256])
    assert gpu_amax(torch.zeros((5, 32), dtype=torch.bfloat16, device="cuda")) == (0.0, 0)
    assert gpu_amax(torch.zeros((0, 32), dtype=torch.bfloat16, device="cuda")) == (0.0, 0)
    bad = to_dev_bf16(x)
    bad[40, 100] = float("inf")
    assert gpu_amax(bad)[1] == fp8.FP8_ERR_NONFINITE


def test_amax_quant_sweep_full_size():
    """The 64 Mi-element log-uniform sweep tensor with planted +-1e5 outliers."""
    x = inputs.quant_sweep()
    a, st = gpu_amax(to_dev_bf16(x))
    assert st == 0 and a == oracle.amax(x)


# ================================================================ fp8_quantize_with_amax
def gpu_quant_given(x_dev, fmt, amax_value, dequant=True):
    rows, cols = x_dev.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    d = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda") if dequant else None
    st = status()
    fp8.fp8_quantize_with_amax(x_dev, fmt, dev_f32(amax_value), q, s, dequant=d, dev_status=st)
    torch.cuda.synchronize()
    return q.cpu().numpy(), np.float32(s.item()), (to_host_u16(d) if dequant else None), int(st.item())


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
@pytest.mark.parametrize("factor", [1.0, 0.25, 4.0, 0.0])
@pytest.mark.parametrize("rows,cols", [(1, 16), (130, 272), (1024, 4096)])
def test_quantize_with_amax_matches_oracle(fmt, factor, rows, cols):
    x = rand_bf16((rows, cols), seed=rows * 7 + cols, spread=2.0)
    a = np.float32(oracle.amax(x) * factor)
    q, s, d, st = gpu_quant_given(to_dev_bf16(x), fmt, a)
    q_ref, s_ref, d_ref = oracle.quantize_with_amax(x, fmt, float(a))
    assert st == 0
    assert s == s_ref, (s, s_ref)
    assert first_mismatch(q, q_ref) is None, first_mismatch(q, q_ref)
    assert first_mismatch(d, d_ref) is None, first_mismatch(d, d_ref)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_quantize_with_amax_strided_and_huge_ratio(fmt):
    """Strided rows, and a tiny given amax so that x / s overflows fp32 for the large
    elements (they must saturate, not turn into NaN)."""
    x = rand_bf16((96, 768), seed=9, spread=3.0)
    g = np.random.default_rng(10)
    # a few huge magnitudes: with the amax floor scale 1e-12 / F_max their x / s is
    # beyond the fp32 range (up to the largest finite bf16)
    for v in (1e30, -1e30, 3.0e38, -3.0e38, 1e24):
        x[g.integers(0, 96), g.integers(128, 640)] = inputs.bf16_bits(np.array([v], np.float32))[0]
    big = to_dev_bf16(x)
    view = big[:, 128:128 + 512]
    for a in (np.float32(oracle.amax(x[:, 128:640])), np.float32(1e-30)):
        q, s, d, st = gpu_quant_given(view, fmt, a)
        q_ref, s_ref, d_ref = oracle.quantize_with_amax(np.ascontiguousarray(x[:, 128:640]), fmt, float(a))
        assert st == 0 and s == s_ref
        assert first_mismatch(q, q_ref) is None, first_mismatch(q, q_ref)
        assert first_mismatch(d, d_ref) is None
    # dense as well
    q, s, d, st = gpu_quant_given(to_dev_bf16(x), fmt, np.float32(1e-30))
    q_ref, s_ref, d_ref = oracle.quantize_with_amax(x, fmt, 1e-30)
    assert st == 0 and s == s_ref and first_mismatch(q, q_ref) is None


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_split_path_equals_tensor_mode_on_gpu(fmt):
    """fp8_amax then fp8_quantize_with_amax gives exactly what fp8_quantize(TENSOR) gives."""
    x = to_dev_bf16(inputs.quant_sweep())
    rows, cols = x.shape
    a = dev_f32(0.0)
    ws = fp8.workspace_for(0, rows, 0, cols, T)
    fp8.fp8_amax(x, a, workspace=ws)
    q1 = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    s1 = torch.empty(1, dtype=torch.float32, device="cuda")
    fp8.fp8_quantize_with_amax(x, fmt, a, q1, s1)
    q2, s2, _ = fp8.empty_quant_outputs(rows, cols, T)
    fp8.fp8_quantize(x, fmt, T, q2, s2, workspace=ws)
    torch.cuda.synchronize()
    assert s1.item() == s2.item() and torch.equal(q1, q2)


def test_quantize_with_amax_empty_and_nonfinite():
    s = torch.full((1,), -1.0, device="cuda")
    q = torch.empty((0, 32), dtype=torch.uint8, device="cuda")
    fp8.fp8_quantize_with_amax(torch.empty((0, 32), dtype=torch.bfloat16, device="cuda"), E4M3, dev_f32(3.0), q, s)
    torch.cuda.synchronize()
    assert s.item() == np.float32(np.float32(3.0) / np.float32(448.0))
    x = rand_bf16((8, 64), seed=1)
    assert gpu_quant_given(to_dev_bf16(x), E4M3, np.float32(np.nan))[3] == fp8.FP8_ERR_NONFINITE
    bad = to_dev_bf16(x)
    bad[2, 5] = float("nan")
    assert gpu_quant_given(bad, E4M3, np.float32(1.0))[3] == fp8.FP8_ERR_NONFINITE


# ================================================================ GEMM epilogue
def quantize_host(x_u16, fmt, mode):
    q, s, _ = oracle.quantize(x_u16, fmt, mode, dequant=False)
    return q, s


def run_ex(qa, sa, am, fa, qb, sb, bm, fb, *, bias=None, want_amax=False, s_y=None, yq_fmt=E4M3, with_y=True,
           ldq=None, yq_offset=0):
    M, K = qa.shape
    N = qb.shape[0]
    a = torch.from_numpy(qa).cuda()
    b = torch.from_numpy(qb).cuda()
    sa_d = torch.from_numpy(np.ascontiguousarray(sa)).cuda()
    sb_d = torch.from_numpy(np.ascontiguousarray(sb)).cuda()
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda") if with_y else None
    bias_d = to_dev_bf16(bias) if bias is not None else None
    amax = dev_f32(0.0) if want_amax else None
    yq = yq_buf = None
    if s_y is not None:
        ldq = ldq or N
        yq_buf = torch.full((max(M, 1) * ldq + yq_offset + 64,), 0xA5, dtype=torch.uint8, device="cuda")
        yq = yq_buf[yq_offset:yq_offset + M * ldq].view(M, ldq)[:, :N] if M > 0 else yq_buf[:0].view(0, N)
    st = status()
    fp8.fp8_scaled_gemm_ex(a, sa_d, am, fa, b, sb_d, bm, fb, y, bias=bias_d, amax=amax, yq=yq,
                           yq_scale=dev_f32(s_y) if s_y is not None else None, yq_fmt=yq_fmt, dev_status=st)
    torch.cuda.synchronize()
    out = {"status": int(st.item())}
    if with_y:
        out["y"] = to_host_u16(y)
    if want_amax:
        out["amax"] = float(amax.item())
    if s_y is not None:
        out["yq"] = yq.cpu().numpy()
        if ldq > N and M > 0:
            pad = yq_buf[yq_offset:yq_offset + M * ldq].view(M, ldq)[:, N:]
            assert torch.all(pad == 0xA5), "FP8 output written outside [M, N]"
    return out


def check_epilogue(x, w, am, bm, *, fa=E4M3, fb=E4M3, yq_fmt=E4M3, seed=0, what="", ldq=None, yq_offset=0):
    """bias + amax + FP8 output against the oracle, then the FP8-only call must give the
    same codes (and the same amax) as the call that also stores Y."""
    qa, sa = quantize_host(x, fa, am)
    qb, sb = quantize_host(w, fb, bm)
    M, N = x.shape[0], w.shape[0]
    g = np.random.default_rng(seed)
    y0, b0 = oracle.gemm_ref_full(qa, sa, am, fa, qb, sb, bm, fb)
    bias = inputs.bf16_bits((g.standard_normal(N) * np.std(y0) * 2).astype(np.float32))
    y_ref, bound = oracle.epilogue_ref(y0, b0, bias)
    # an output scale from half the reference amax: the largest outputs saturate
    s_y = oracle.scale_from_amax(float(np.max(np.abs(y_ref))) / 2, yq_fmt)
    r = run_ex(qa, sa, am, fa, qb, sb, bm, fb, bias=bias, want_amax=True, s_y=s_y, yq_fmt=yq_fmt, ldq=ldq,
               yq_offset=yq_offset)
    assert r["status"] == 0, r["status"]
    assert_gemm_close(r["y"], y_ref, bound, what + " y")
    yv = bf16_bits_to_f64(r["y"])
    assert r["amax"] == float(np.max(np.abs(yv))), (r["amax"], np.max(np.abs(yv)))
    lim = 1e-3 * bound + oracle.bf16_ulp(y_ref)
    assert np.max(np.abs(y_ref) - lim) <= r["amax"] <= np.max(np.abs(y_ref) + lim)
    lo, hi = oracle.requant_interval(y_ref, lim, s_y, yq_fmt)
    cv = oracle.decode_table(yq_fmt)[r["yq"]]
    bad = ~((cv >= lo) & (cv <= hi))
    assert not bad.any(), f"{what}: {int(bad.sum())} FP8 outputs outside the admissible codes, first " \
                          f"{np.argwhere(bad)[:4].tolist()}"
    r2 = run_ex(qa, sa, am, fa, qb, sb, bm, fb, bias=bias, want_amax=True, s_y=s_y, yq_fmt=yq_fmt, with_y=False,
                ldq=ldq, yq_offset=yq_offset)
    assert r2["status"] == 0 and r2["amax"] == r["amax"]
    assert first_mismatch(r2["yq"], r["yq"]) is None
    return r, s_y


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (1, 16, 32), (130, 264, 512), (300, 520, 1024)])
@pytest.mark.parametrize("am,bm", [(T, T), (R, R)])
@pytest.mark.parametrize("yq_fmt", [E4M3, E5M2])
def test_rowscale_epilogue(M, N, K, am, bm, yq_fmt):
    x = rand_bf16((M, K), seed=M + K, spread=1.0)
    w = rand_bf16((N, K), seed=N + K, std=0.02)
    check_epilogue(x, w, am, bm, yq_fmt=yq_fmt, seed=M, what=f"rowscale {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (130, 264, 1024), (300, 264, 512), (512, 384, 256)])
def test_block_epilogue(M, N, K):
    x = rand_bf16((M, K), seed=M * 3 + K, spread=1.0)
    w = rand_bf16((N, K), seed=N * 3 + K, std=0.02)
    check_epilogue(x, w, B1, B128, seed=K, what=f"block {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (130, 264, 1056)])
def test_mx_epilogue(M, N, K):
    x = rand_bf16((M, K), seed=M * 5 + K, spread=1.0)
    w = rand_bf16((N, K), seed=N * 5 + K, std=0.02)
    check_epilogue(x, w, MX, MX, seed=N, what=f"mx {M}x{N}x{K}")


def test_epilogue_ragged_fp8_stride_and_offset():
    """FP8 output rows that are not 16-byte aligned take the byte-store path."""
    x = rand_bf16((257, 512), seed=71)
    w = rand_bf16((200, 512), seed=72, std=0.02)
    check_epilogue(x, w, R, R, ldq=203, yq_offset=5, what="ragged ldq")


@pytest.mark.parametrize("am,bm,M", [(T, T, 64), (T, T, 300), (B1, B128, 128), (B1, B128, 384), (MX, MX, 128)])
def test_epilogue_exact_integer(am, bm, M):
    """Small-integer codes, unit scales and an integer bias: y, amax and the FP8 output
    codes are exact, so they must equal the oracle bit for bit."""
    g = np.random.default_rng(81 + M)
    N, K = 256, 128
    a_int = g.integers(-2, 3, (M, K)).astype(np.float32)
    b_int = g.integers(-2, 3, (N, K)).astype(np.float32)
    qa = oracle.encode(a_int, E4M3).reshape(M, K)
    qb = oracle.encode(b_int, E4M3).reshape(N, K)
    if am == MX:
        sa = np.full((M, K // 32), 127, np.uint8)
        sb = np.full((N, K // 32), 127, np.uint8)
    elif am == B1:
        sa = np.ones((M, K // 128), np.float32)
        sb = np.ones((N // 128, K // 128), np.float32)
    else:
        sa = np.ones(1, np.float32)
        sb = np.ones(1, np.float32)
    bias = inputs.bf16_bits(g.integers(-50, 51, N).astype(np.float32))
    y0, b0 = oracle.gemm_ref_full(qa, sa, am, E4M3, qb, sb, bm, E4M3)
    y_ref, _ = oracle.epilogue_ref(y0, b0, bias)
    assert np.max(np.abs(y_ref)) < 256          # exact in bf16
    s_y = oracle.scale_from_amax(float(np.max(np.abs(y_ref))), E4M3)
    r = run_ex(qa, sa, am, E4M3, qb, sb, bm, E4M3, bias=bias, want_amax=True, s_y=s_y)
    assert r["status"] == 0
    assert np.array_equal(bf16_bits_to_f64(r["y"]), y_ref)
    assert r["amax"] == float(np.max(np.abs(y_ref)))
    q_ref = oracle.quant_scaled(y_ref.astype(np.float32), s_y, E4M3).reshape(M, N)
    assert first_mismatch(r["yq"], q_ref) is None, first_mismatch(r["yq"], q_ref)


def test_epilogue_zero_k_and_bias_only():
    """K = 0: y = bf16(bias), amax = max|bias|, codes of bias / s_y."""
    M, N = 70, 100
    g = np.random.default_rng(5)
    bias = inputs.bf16_bits((g.standard_normal(N) * 3).astype(np.float32))
    bv = oracle.bf16_to_f32(bias)
    s_y = oracle.scale_from_amax(float(np.max(np.abs(bv))), E5M2)
    qa = np.zeros((M, 0), np.uint8)
    qb = np.zeros((N, 0), np.uint8)
    one = np.ones(1, np.float32)
    r = run_ex(qa, one, T, E4M3, qb, one, T, E4M3, bias=bias, want_amax=True, s_y=s_y, yq_fmt=E5M2)
    assert r["status"] == 0
    assert np.array_equal(r["y"], np.broadcast_to(bias, (M, N)))
    assert r["amax"] == float(np.max(np.abs(bv)))
    q_ref = oracle.quant_scaled(bv, s_y, E5M2)
    assert np.array_equal(r["yq"], np.broadcast_to(q_ref, (M, N)))


def test_epilogue_bias_only_and_amax_only():
    x = rand_bf16((300, 512), seed=91)
    w = rand_bf16((264, 512), seed=92, std=0.02)
    qa, sa = quantize_host(x, E4M3, R)
    qb, sb = quantize_host(w, E4M3, R)
    y0, b0 = oracle.gemm_ref_full(qa, sa, R, E4M3, qb, sb, R, E4M3)
    bias = inputs.bf16_bits(np.linspace(-2, 2, 264).astype(np.float32))
    r = run_ex(qa, sa, R, E4M3, qb, sb, R, E4M3, bias=bias)
    y_ref, bound = oracle.epilogue_ref(y0, b0, bias)
    assert r["status"] == 0
    assert_gemm_close(r["y"], y_ref, bound, "bias only")
    r = run_ex(qa, sa, R, E4M3, qb, sb, R, E4M3, want_amax=True)
    assert r["amax"] == float(np.max(np.abs(bf16_bits_to_f64(r["y"]))))
    assert_gemm_close(r["y"], y0, b0, "amax only")


def test_epilogue_bad_arguments_and_bad_scale():
    qa = np.zeros((128, 64), np.uint8)
    qb = np.zeros((128, 64), np.uint8)
    one = torch.ones(1, device="cuda")
    a = torch.from_numpy(qa).cuda()
    b = torch.from_numpy(qb).cuda()
    y = torch.empty((128, 128), dtype=torch.bfloat16, device="cuda")
    yq = torch.empty((128, 128), dtype=torch.uint8, device="cuda")
    with pytest.raises(fp8.FP8Error) as e:            # FP8 output without its scale
        fp8.fp8_scaled_gemm_ex(a, one, T, E4M3, b, one, T, E4M3, y, yq=yq)
    assert e.value.status == fp8.FP8_ERR_INVALID_ARG
    with pytest.raises(fp8.FP8Error) as e:            # no output at all
        fp8.fp8_scaled_gemm_ex(a, one, T, E4M3, b, one, T, E4M3, None)
    assert e.value.status == fp8.FP8_ERR_INVALID_ARG
    bias = torch.zeros(129, dtype=torch.bfloat16, device="cuda")[1:]
    with pytest.raises(fp8.FP8Error) as e:            # bias not 16-byte aligned
        fp8.fp8_scaled_gemm_ex(a, one, T, E4M3, b, one, T, E4M3, y, bias=bias)
    assert e.value.status == fp8.FP8_ERR_ALIGNMENT
    with pytest.raises(fp8.FP8Error) as e:            # bad output format
        fp8.fp8_scaled_gemm_ex(a, one, T, E4M3, b, one, T, E4M3, y, yq=yq, yq_scale=one, yq_fmt=7)
    assert e.value.status == fp8.FP8_ERR_INVALID_ARG
    st = status()
    fp8.fp8_scaled_gemm_ex(a, one, T, E4M3, b, one, T, E4M3, y, yq=yq, yq_scale=dev_f32(0.0), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == fp8.FP8_ERR_INVALID_ARG


# ================================================================ chains and full size
def test_linear_forward_ex_chain_uses_output_amax():
    """Two layers: the first GEMM's output amax feeds the second layer's per-tensor cast,
    which must then equal fp8_quantize(TENSOR) of the stored Y bit for bit."""
    x = to_dev_bf16(rand_bf16((512, 1024), seed=101, spread=1.0))
    w_host = rand_bf16((768, 1024), seed=102, std=0.02)
    qw, sw = quantize_host(w_host, E4M3, R)
    w = torch.from_numpy(qw).cuda()
    sw_d = torch.from_numpy(sw).cuda()
    bias = to_dev_bf16(inputs.bf16_bits(np.linspace(-1, 1, 768).astype(np.float32)))
    y = torch.empty((512, 768), dtype=torch.bfloat16, device="cuda")
    amax = dev_f32(0.0)
    ws = fp8.workspace_for(2, 512, 768, 1024, R)
    st = status()
    fp8.fp8_linear_forward_ex(x, E4M3, R, w, sw_d, R, E4M3, y, ws, bias=bias, amax=amax, dev_status=st)
    q1 = torch.empty((512, 768), dtype=torch.uint8, device="cuda")
    s1 = torch.empty(1, device="cuda")
    fp8.fp8_quantize_with_amax(y, E4M3, amax, q1, s1, dev_status=st)
    q2, s2, _ = fp8.empty_quant_outputs(512, 768, T)
    fp8.fp8_quantize(y, E4M3, T, q2, s2, workspace=fp8.workspace_for(0, 512, 0, 768, T))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert amax.item() == y.float().abs().max().item()
    assert s1.item() == s2.item() and torch.equal(q1, q2)
    # and Y itself against the oracle (X quantised by the oracle, per token)
    qa, sa = quantize_host(to_host_u16(x), E4M3, R)
    y0, b0 = oracle.gemm_ref_full(qa, sa, R, E4M3, qw, sw, R, E4M3)
    y_ref, bound = oracle.epilogue_ref(y0, b0, to_host_u16(bias))
    assert_gemm_close(to_host_u16(y), y_ref, bound, "linear_forward_ex")


def test_fp8_output_matches_requantised_y_full_size():
    """The 4096 x 28672 x 8192 per-token / per-channel layer with bias: the FP8-only output
    equals fp8_quantize_with_amax of the stored Y under the same scale, the output amax is
    max|Y|, and Y matches the oracle at sampled outputs."""
    x_u16, w_u16 = inputs.llama70b_prefill()
    M, K = x_u16.shape
    N = w_u16.shape[0]
    qa, sa = quantize_host(x_u16, E4M3, R)
    qb, sb = quantize_host(w_u16, E4M3, R)
    g = np.random.default_rng(7)
    bias_u16 = inputs.bf16_bits((g.standard_normal(N) * 0.5).astype(np.float32))
    a = torch.from_numpy(qa).cuda()
    b = torch.from_numpy(qb).cuda()
    sa_d, sb_d = torch.from_numpy(sa).cuda(), torch.from_numpy(sb).cuda()
    bias = to_dev_bf16(bias_u16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    amax = dev_f32(0.0)
    st = status()
    fp8.fp8_scaled_gemm_ex(a, sa_d, R, E4M3, b, sb_d, R, E4M3, y, bias=bias, amax=amax, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert amax.item() == y.float().abs().max().item()
    # sampled outputs against the oracle; the output scale comes from their amax
    pm = np.concatenate([g.integers(0, M, 20000), np.full(256, M - 1)])
    pn = np.concatenate([g.integers(0, N, 20000), np.arange(N - 256, N)])
    y0, b0 = oracle.gemm_ref_points(qa, sa, R, E4M3, qb, sb, R, E4M3, pm, pn)
    y_ref, bound = oracle.epilogue_ref(y0, b0, bias_u16[pn])
    assert_gemm_close(to_host_u16(y)[pm, pn], y_ref, bound, "llama70b_prefill with bias")
    a_ref = np.float32(np.max(np.abs(y_ref)))
    s_y = oracle.scale_from_amax(float(a_ref), E4M3)
    # the stored Y requantised by the cast kernel with that scale ...
    s_gpu = torch.empty(1, device="cuda")
    q_ref_gpu = torch.empty((M, N), dtype=torch.uint8, device="cuda")
    fp8.fp8_quantize_with_amax(y, E4M3, dev_f32(a_ref), q_ref_gpu, s_gpu)
    torch.cuda.synchronize()
    assert np.float32(s_gpu.item()) == np.float32(s_y)
    # ... equals the FP8-only epilogue output under the same scale
    yq = torch.empty((M, N), dtype=torch.uint8, device="cuda")
    amax2 = dev_f32(0.0)
    fp8.fp8_scaled_gemm_ex(a, sa_d, R, E4M3, b, sb_d, R, E4M3, None, bias=bias, amax=amax2, yq=yq,
                           yq_scale=dev_f32(s_y), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and amax2.item() == amax.item()
    assert torch.equal(yq, q_ref_gpu)
    lim = 1e-3 * bound + oracle.bf16_ulp(y_ref)
    lo, hi = oracle.requant_interval(y_ref, lim, s_y, E4M3)
    cv = oracle.decode_table(E4M3)[yq.cpu().numpy()[pm, pn]]
    assert np.all((cv >= lo) & (cv <= hi))
