"""GPU parity of the weight-only FP8 linear (fp8_weight_only_linear) through the C ABI.

X stays BF16; the weight is FP8 codes with a per-tensor or per-row scale (quantised
by the oracle here, so the test does not lean on the GPU quantiser).  Reference: the
oracle's fp64 sum of x times the decoded, scaled weight, under the usual acceptance
rule |y - y_ref| <= 1e-3 * sum_k |terms| + 1 bf16 ulp; exact integer cases are
compared bit for bit.  Up to 3 tokens the CUDA-core matrix-vector kernel runs,
above that the tensor-core one; the token counts cover both sides of the switch.
The shapes hit one-unit and uneven per-SM ranges, several chunks per CTA, ragged N
(not a multiple of the 8-row groups) and K (a last stage with fewer K blocks, a
half-empty last K block, K below one 128-code step) and token counts up to the
maximum."""
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
T, R = fp8.FP8_SCALE_TENSOR, fp8.FP8_SCALE_ROW


def rand_bf16(shape, seed, std=1.0, spread=0.0):
    g = np.random.default_rng(seed)
    x = g.standard_normal(shape).astype(np.float32) * np.float32(std)
    if spread:
        x *= np.exp(g.standard_normal((shape[0], 1)) * spread).astype(np.float32)
    return inputs.bf16_bits(x)


def run_wo(x_u16, qw, sw, mode, fmt, ldx=None, ldy=None):
    M, K = x_u16.shape
    N = qw.shape[0]
    ldx = ldx or K
    xb = torch.zeros((max(M, 1), ldx), dtype=torch.bfloat16, device="cuda")
    if M:
        xb[:M, :K] = to_dev_bf16(x_u16)
    x = xb[:M, :K]
    ldy = ldy or N
    yb = torch.full((max(M, 1), ldy), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = yb[:M, :N]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8.fp8_weight_only_linear(x, torch.from_numpy(qw).cuda(), torch.from_numpy(np.ascontiguousarray(sw)).cuda(),
                               mode, fmt, y, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    out = to_host_u16(yb)
    if ldy > N and M:
        assert np.all(np.isnan(bf16_bits_to_f64(out[:M, N:]))), "wrote outside [M, N]"
    return out[:M, :N]


def check(M, N, K, mode, fmt, seed, ldx=None, ldy=None):
    x = rand_bf16((M, K), seed, spread=1.0)
    w = rand_bf16((N, K), seed + 1, std=0.02, spread=0.5)
    qw, sw, _ = oracle.quantize(w, fmt, mode, dequant=False)
    y = run_wo(x, qw, sw, mode, fmt, ldx, ldy)
    y_ref, bound = oracle.weight_only_ref(x, qw, sw, mode, fmt)
    assert_gemm_close(y, y_ref, bound, f"weight-only {M}x{N}x{K} mode {mode} fmt {fmt}")


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 9, 16, 33, 64])
@pytest.mark.parametrize("N,K", [(16, 128), (200, 512), (2368, 256), (3000, 640), (1000, 1040), (300, 16),
                                 (20000, 1152), (13, 48), (4099, 400)])
def test_weight_only_shapes(M, N, K):
    check(M, N, K, R, E4M3, seed=M * 13 + N + K)


@pytest.mark.parametrize("M", [4, 16])
@pytest.mark.parametrize("mode", [T, R])
@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_weight_only_modes_and_formats(M, mode, fmt):
    check(M, 1500, 768, mode, fmt, seed=7 + fmt + M)


@pytest.mark.parametrize("M", [3, 9])
def test_weight_only_strides(M):
    check(M, 700, 512, R, E4M3, seed=3, ldx=512 + 24, ldy=700 + 40)
    check(M, 700, 512, R, E4M3, seed=4, ldy=703)


@pytest.mark.parametrize("M", [1, 6, 16])
def test_weight_only_exact_integer(M):
    """Integer activations (exact in bf16) and integer codes with unit scale: exact."""
    g = np.random.default_rng(61 + M)
    N, K = 512, 256
    x_int = g.integers(-2, 3, (M, K)).astype(np.float32)
    w_int = g.integers(-2, 3, (N, K)).astype(np.float32)
    x = inputs.bf16_bits(x_int)
    qw = oracle.encode(w_int, E4M3).reshape(N, K)
    y = run_wo(x, qw, np.ones(1, np.float32), T, E4M3)
    y_ref, _ = oracle.weight_only_ref(x, qw, np.ones(1, np.float32), T, E4M3)
    assert np.max(np.abs(y_ref)) < 256
    assert np.array_equal(bf16_bits_to_f64(y), y_ref)


def test_weight_only_empty_zero_k_and_bad_args():
    w = torch.zeros((32, 64), dtype=torch.uint8, device="cuda")
    s = torch.ones(1, device="cuda")
    y = torch.full((4, 32), 1.0, dtype=torch.bfloat16, device="cuda")
    fp8.fp8_weight_only_linear(torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda"), w, s, T, E4M3, y[:0])
    fp8.fp8_weight_only_linear(torch.zeros((4, 0), dtype=torch.bfloat16, device="cuda"),
                               torch.zeros((32, 0), dtype=torch.uint8, device="cuda"), s, T, E4M3, y)
    torch.cuda.synchronize()
    assert torch.all(y == 0)
    x = torch.zeros((65, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_weight_only_linear(x, w, s, T, E4M3, torch.empty((65, 32), dtype=torch.bfloat16, device="cuda"))
    assert e.value.status == fp8.FP8_ERR_INVALID_ARG
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_weight_only_linear(x[:4], w, s, fp8.FP8_SCALE_MX32, E4M3, y)
    assert e.value.status == fp8.FP8_ERR_INVALID_ARG
    xs = torch.zeros((4, 68), dtype=torch.bfloat16, device="cuda")[:, :64]     # row stride 68: not 16-byte rows
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_weight_only_linear(xs, w, s, T, E4M3, y)
    assert e.value.status == fp8.FP8_ERR_ALIGNMENT


@pytest.mark.parametrize("M", [1, 4, 8, 16, 64])
def test_weight_only_llama70b_layer_full_size(M):
    """M tokens against the whole 28672 x 8192 weight (per-channel scales), every output
    of 2,048 sampled weight rows against the oracle."""
    x, w = inputs.llama70b_prefill(M=M)
    qw, sw, _ = oracle.quantize(w, E4M3, R, dequant=False)
    y = run_wo(x, qw, sw, R, E4M3)
    cols = np.sort(np.random.default_rng(5).choice(qw.shape[0], 2048, replace=False))
    y_ref, bound = oracle.weight_only_ref(x, qw[cols], sw[cols], R, E4M3)
    assert_gemm_close(y[:, cols], y_ref, bound, f"weight-only llama70b M={M}")


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 16, 64])
def test_weight_only_every_code_decodes_exactly(M, fmt):
    """Every one of the 256 codes through the weight decode of both kernels.  X is one-hot
    (token m picks column m), so y[m, n] is the decoded code w[n, m] itself, exact in
    bf16 (every FP8 value is a bf16 value): the finite codes fill rows M codes a row,
    subnormals and both zeros included, and are compared bit for bit with the oracle's
    decode table.  A NaN or Inf code (E5M2 also has Inf) gets a row of its own at column
    0: token 0 reads the code times 1, every other token 0 times the code (NaN)."""
    table = oracle.decode_table(fmt)
    codes = np.arange(256)
    finite = codes[np.isfinite(table)]
    special = codes[~np.isfinite(table)]
    K = max(64, -(-M // 16) * 16)
    nf = -(-len(finite) // M)
    w = np.zeros((nf + len(special), K), np.uint8)
    flat = np.zeros(nf * M, np.int64)
    flat[:len(finite)] = finite
    w[:nf, :M] = flat.reshape(nf, M)
    w[nf:, 0] = special
    x = np.zeros((M, K), np.float32)
    x[np.arange(M), np.arange(M)] = 1.0
    y = bf16_bits_to_f64(run_wo(inputs.bf16_bits(x), w, np.ones(1, np.float32), T, fmt))
    want = table[w[:nf, :M]].T                       # [M, nf]
    assert np.array_equal(y[:, :nf], want), f"finite codes, fmt {fmt}, M {M}"
    got_s = y[:, nf:]
    assert np.array_equal(got_s[0], table[special], equal_nan=True), f"special codes, token 0, fmt {fmt}"
    assert np.all(np.isnan(got_s[1:])), f"special codes times 0, fmt {fmt}"
