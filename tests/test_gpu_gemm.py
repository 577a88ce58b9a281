"""GPU parity of fp8_scaled_gemm and fp8_linear_forward (through the C ABI).

Reference: the oracle's fp64 sum of dequantised products; acceptance rule
|y - y_ref| <= 1e-3 * sum_k |terms| + 1 bf16 ulp(y_ref).  Small problems are
checked at every output; full-size problems at sampled outputs against the
oracle plus every output against an fp32 torch matmul of the dequantised
operands (a library second opinion, with the same rule)."""
import numpy as np
import pytest
import torch

import oracle
from fp8_dynamic_scaled_b200 import inputs
from gpu_util import assert_gemm_close, bf16_bits_to_f64, to_dev_bf16, to_host_u16

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
import fp8_dynamic_scaled_b200.binding as fp8  # noqa: E402

E4M3, E5M2 = fp8.FP8_E4M3, fp8.FP8_E5M2
T, R, B1, B128, MX = (fp8.FP8_SCALE_TENSOR, fp8.FP8_SCALE_ROW, fp8.FP8_SCALE_BLOCK_1x128,
                      fp8.FP8_SCALE_BLOCK_128x128, fp8.FP8_SCALE_MX32)


def quantize_host(x_u16, fmt, mode):
    """Operands for the GEMM come from the oracle's quantizer (the GEMM test must not
    depend on the GPU quantizer being right)."""
    q, s, _ = oracle.quantize(x_u16, fmt, mode, dequant=False)
    return q, s


def gemm_gpu(qa, sa, am, fa, qb, sb, bm, fb, ldy=None):
    M, K = qa.shape
    N = qb.shape[0]
    ldy = ldy or N
    a = torch.from_numpy(qa).cuda()
    b = torch.from_numpy(qb).cuda()
    sa_d = torch.from_numpy(np.ascontiguousarray(sa)).cuda()
    sb_d = torch.from_numpy(np.ascontiguousarray(sb)).cuda()
    ybuf = torch.full((max(M, 1), ldy), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = ybuf[:M, :N]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8.fp8_scaled_gemm(a, sa_d, am, fa, b, sb_d, bm, fb, y, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, f"dev_status {int(st.item())}"
    out = to_host_u16(ybuf)
    if ldy > N and M > 0:
        assert np.all(out[:M, N:] == to_host_u16(torch.full((1,), float("nan"), dtype=torch.bfloat16))[0]), \
            "GEMM wrote outside [M, N]"
    return out[:M, :N]


def check_full(x, w, am, bm, fa=E4M3, fb=E4M3, what="", ldy=None):
    qa, sa = quantize_host(x, fa, am)
    qb, sb = quantize_host(w, fb, bm)
    y = gemm_gpu(qa, sa, am, fa, qb, sb, bm, fb, ldy=ldy)
    y_ref, bound = oracle.gemm_ref_full(qa, sa, am, fa, qb, sb, bm, fb)
    assert_gemm_close(y, y_ref, bound, what)
    return y, y_ref


def rand_bf16(shape, seed, std=1.0, lognormal_rows=False):
    g = np.random.default_rng(seed)
    x = g.standard_normal(shape).astype(np.float32) * np.float32(std)
    if lognormal_rows:
        x *= np.exp(g.standard_normal((shape[0], 1))).astype(np.float32)
    return inputs.bf16_bits(x)


# ---------------------------------------------------------------- small, every output
def test_linear_small_config_tensor_scaling():
    """X [128,256] with a planted 400.0, W [256,256]: per-tensor current X, static W."""
    x, w = inputs.linear_small()
    check_full(x, w, T, T, what="linear_small")


SHAPES = [(128, 256, 256), (1, 8, 16), (130, 260, 272), (257, 520, 1040), (300, 700, 512)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("am,bm", [(T, T), (R, R), (T, R), (R, T)])
def test_rowscale_shapes(M, N, K, am, bm):
    x = rand_bf16((M, K), seed=M + N + K, lognormal_rows=True)
    w = rand_bf16((N, K), seed=M * N + K, std=0.02, lognormal_rows=True)
    check_full(x, w, am, bm, what=f"rowscale {M}x{N}x{K} {am}/{bm}")


@pytest.mark.parametrize("fa,fb", [(E5M2, E5M2), (E4M3, E5M2), (E5M2, E4M3)])
def test_rowscale_e5m2_operands(fa, fb):
    x = rand_bf16((257, 512), seed=1, lognormal_rows=True)
    w = rand_bf16((300, 512), seed=2, std=0.02)
    check_full(x, w, R, R, fa=fa, fb=fb, what=f"formats {fa}/{fb}")


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (130, 260, 1040), (257, 520, 2048), (64, 128, 128),
                                   (256, 128, 128), (300, 384, 640), (513, 200, 1024), (1024, 1152, 512)])
def test_block_scaled_shapes(M, N, K):
    g = np.random.default_rng(M + K)
    x = g.standard_normal((M, K)).astype(np.float32)
    x *= np.repeat(np.exp(g.standard_normal((M, -(-K // 128)))).astype(np.float32), 128, axis=1)[:, :K]
    w = g.standard_normal((N, K)).astype(np.float32)
    fw = np.exp(g.standard_normal((-(-N // 128), -(-K // 128)))).astype(np.float32)
    w *= np.repeat(np.repeat(fw, 128, axis=0), 128, axis=1)[:N, :K]
    check_full(inputs.bf16_bits(x), inputs.bf16_bits(w), B1, B128, what=f"block {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (130, 260, 1056), (257, 520, 2048), (1, 16, 32)])
def test_mx_shapes(M, N, K):
    g = np.random.default_rng(M * 3 + K)
    x = (g.standard_normal((M, K)) * np.exp2(g.integers(-12, 12, (M, K // 32))).repeat(32, axis=1)).astype(np.float32)
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    check_full(inputs.bf16_bits(x), inputs.bf16_bits(w), MX, MX, what=f"mx {M}x{N}x{K}")


def test_output_row_stride_and_edges():
    x = rand_bf16((130, 512), seed=7)
    w = rand_bf16((264, 512), seed=8, std=0.02)
    check_full(x, w, R, R, what="ldy", ldy=264 + 40)


def test_exact_integer_gemm_is_bit_exact():
    """Small-integer codes with unit scales: every partial sum is an integer below 2^24,
    so the bf16 result must equal the exactly rounded integer result."""
    g = np.random.default_rng(5)
    M, N, K = 256, 512, 1024
    ai = g.integers(-4, 5, (M, K))
    bi = g.integers(-4, 5, (N, K))
    qa = oracle.encode(ai.astype(np.float32), E4M3).reshape(M, K)
    qb = oracle.encode(bi.astype(np.float32), E4M3).reshape(N, K)
    one = np.ones(1, np.float32)
    y = gemm_gpu(qa, one, T, E4M3, qb, one, T, E4M3)
    exact = (ai @ bi.T).astype(np.float32)
    assert np.array_equal(y, oracle.f32_to_bf16(exact).reshape(M, N))


def test_identity_weight():
    K = 512
    x = rand_bf16((300, K), seed=9)
    w = inputs.bf16_bits(np.eye(K, dtype=np.float32))
    check_full(x, w, R, T, what="identity")


def test_zero_k_writes_zeros_and_empty_is_noop():
    a = torch.zeros((5, 0), dtype=torch.uint8, device="cuda")
    b = torch.zeros((7, 0), dtype=torch.uint8, device="cuda")
    s = torch.ones(1, device="cuda")
    y = torch.full((5, 8), 3.0, dtype=torch.bfloat16, device="cuda")[:, :7]
    fp8.fp8_scaled_gemm(a, s, T, E4M3, b, s, T, E4M3, y)
    torch.cuda.synchronize()
    assert torch.all(y == 0)
    y2 = torch.zeros((0, 8), dtype=torch.bfloat16, device="cuda")
    fp8.fp8_scaled_gemm(torch.zeros((0, 16), dtype=torch.uint8, device="cuda"), s, T, E4M3,
                        torch.zeros((8, 16), dtype=torch.uint8, device="cuda"), s, T, E4M3, y2)


def test_gemm_rejects_bad_mode_pairs():
    a = torch.zeros((128, 128), dtype=torch.uint8, device="cuda")
    s = torch.ones(128, device="cuda")
    y = torch.empty((128, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fp8.FP8Error):
        fp8.fp8_scaled_gemm(a, s, B1, E4M3, a, s, R, E4M3, y)
    with pytest.raises(fp8.FP8Error):
        fp8.fp8_scaled_gemm(a, s, MX, E4M3, a, s, MX, E5M2, y)


# ---------------------------------------------------------------- full sizes
def _points(M, N, n, seed):
    g = np.random.default_rng(seed)
    pm = np.concatenate([g.integers(0, M, n), [0, M - 1, M - 1, 0]])
    pn = np.concatenate([g.integers(0, N, n), [0, N - 1, 0, N - 1]])
    return pm, pn


def full_size_check(x, w, am, bm, what, npts=65536):
    """The whole GPU path (fp8_quantize of X and W, then fp8_scaled_gemm) against the
    oracle's own quantisation and fp64 GEMM at 65,536 sampled outputs (plus the four
    corners) and at every output of the first and last 128 rows; every output is also
    checked against an fp32 torch matmul of the oracle's dequantised operands."""
    M, K = x.shape
    N = w.shape[0]
    qa, sa, _ = fp8.empty_quant_outputs(M, K, am)
    qb, sb, _ = fp8.empty_quant_outputs(N, K, bm)
    fp8.fp8_quantize(to_dev_bf16(x), E4M3, am, qa, sa, workspace=fp8.workspace_for(0, M, 0, K, am))
    fp8.fp8_quantize(to_dev_bf16(w), E4M3, bm, qb, sb, workspace=fp8.workspace_for(0, N, 0, K, bm))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8.fp8_scaled_gemm(qa, sa, am, E4M3, qb, sb, bm, E4M3, y, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    del qa, sa, qb, sb
    # the oracle quantises the same inputs itself
    qa_h, sa_h = quantize_host(x, E4M3, am)
    qb_h, sb_h = quantize_host(w, E4M3, bm)
    pm, pn = _points(M, N, npts, seed=M + N)
    y_ref, bound = oracle.gemm_ref_points(qa_h, sa_h, am, E4M3, qb_h, sb_h, bm, E4M3, pm, pn)
    y_h = to_host_u16(y)
    assert_gemm_close(y_h[pm, pn], y_ref, bound, what + " (oracle points)")
    band = np.unique(np.concatenate([np.arange(0, min(128, M)), np.arange(max(0, M - 128), M)]))
    y_band, b_band = oracle.gemm_ref_rows(qa_h, sa_h, am, E4M3, qb_h, sb_h, bm, E4M3, band)
    assert_gemm_close(y_h[band], y_band, b_band, what + " (oracle, first and last 128 rows)")
    del y_band, b_band
    # every output against a dequantised fp32 matmul of the oracle's operands (chunked over rows)
    qa, sa = torch.from_numpy(qa_h).cuda(), torch.from_numpy(np.ascontiguousarray(sa_h)).cuda()
    qb, sb = torch.from_numpy(qb_h).cuda(), torch.from_numpy(np.ascontiguousarray(sb_h)).cuda()

    def deq(q, s, mode, rows):
        v = q.view(torch.float8_e4m3fn).float()
        if mode == T:
            return v * s[0]
        if mode == R:
            return v * s[:, None]
        if mode == B1:
            return v * s.repeat_interleave(128, dim=1)[:, :K]
        if mode == B128:
            return v * s.repeat_interleave(128, dim=0).repeat_interleave(128, dim=1)[:rows, :K]
        return v * torch.exp2(s.float() - 127).repeat_interleave(32, dim=1)

    wb = deq(qb, sb, bm, N)
    wa = wb.abs()
    for r0 in range(0, M, 2048):
        r1 = min(M, r0 + 2048)
        xa = deq(qa[r0:r1], sa if am == T else sa[r0:r1], am, r1 - r0)
        ref = (xa @ wb.T).double()
        bnd = (xa.abs() @ wa.T).double()
        got = y[r0:r1].double()
        # the fp32 reference itself carries up to ~K * 2^-24 relative error of the bound
        lim = 1e-3 * bnd + torch.exp2(torch.floor(torch.log2(ref.abs().clamp_min(2.0 ** -126))) - 7) \
            + 1e-5 * bnd
        bad = (got - ref).abs() > lim
        assert not bool(bad.any()), f"{what}: {int(bad.sum())} outputs off the fp32 reference in rows {r0}..{r1}"


def test_llama70b_prefill_gemm_full_size():
    x, w = inputs.llama70b_prefill()
    full_size_check(x, w, R, R, "llama70b prefill per-token x per-channel")


def test_block_scaled_gemm_full_size():
    x, w = inputs.block_scaled()
    full_size_check(x, w, B1, B128, "block-scaled 1x128 x 128x128")


def test_mx_gemm_full_size():
    x, w = inputs.mx_delayed()
    full_size_check(x, w, MX, MX, "MXFP8")


# ---------------------------------------------------------------- fused linear forward
@pytest.mark.parametrize("x_mode,w_mode", [(T, T), (R, R), (B1, B128), (MX, MX)])
def test_linear_forward_matches_quantize_then_gemm(x_mode, w_mode):
    M, N, K = 257, 520, 1024
    x = rand_bf16((M, K), seed=21, lognormal_rows=True)
    w = rand_bf16((N, K), seed=22, std=0.02)
    qb, sb = quantize_host(w, E4M3, w_mode)
    xd = to_dev_bf16(x)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = fp8.workspace_for(2, M, N, K, x_mode)
    fp8.fp8_linear_forward(xd, E4M3, x_mode, torch.from_numpy(qb).cuda(), torch.from_numpy(sb).cuda(), w_mode, E4M3,
                           y, ws)
    torch.cuda.synchronize()
    qa, sa = quantize_host(x, E4M3, x_mode)
    y_ref, bound = oracle.gemm_ref_full(qa, sa, x_mode, E4M3, qb, sb, w_mode, E4M3)
    assert_gemm_close(to_host_u16(y), y_ref, bound, f"linear {x_mode}/{w_mode}")


def test_linear_forward_delayed_steps():
    M, N, K = 256, 512, 512
    w = rand_bf16((N, K), seed=23, std=0.02)
    qb, sb = quantize_host(w, E4M3, T)
    hist = fp8.History(16)
    ring = np.zeros(16, np.float32)
    ws = fp8.workspace_for(2, M, N, K, fp8.FP8_SCALE_DELAYED)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    wq, ws_ = torch.from_numpy(qb).cuda(), torch.from_numpy(sb).cuda()
    for t in range(18):
        x = inputs.delayed_step_input(t, M=M, K=K)
        fp8.fp8_linear_forward(to_dev_bf16(x), E4M3, fp8.FP8_SCALE_DELAYED, wq, ws_, T, E4M3, y, ws, hist=hist)
        torch.cuda.synchronize()
        qa, s_t, _, _ = oracle.delayed_step(x, E4M3, ring, t)
        y_ref, bound = oracle.gemm_ref_full(qa, np.array([s_t], np.float32), T, E4M3, qb, sb, T, E4M3)
        assert_gemm_close(to_host_u16(y), y_ref, bound, f"delayed linear step {t}")
    assert np.array_equal(hist.ring.cpu().numpy(), ring)
