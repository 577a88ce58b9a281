"""GPU parity of the few-token (decode-shaped, M <= 128) GEMM path through the C ABI.

Calls with M <= 64 go to the weight-streaming kernel: W's rows are split over all
SMs in 16-row units and done in chunks of <= 128 rows, two or four K blocks per
stage, so the shapes below hit one-unit ranges, uneven ranges, several chunks per
CTA, ragged N and K, a last stage with fewer K blocks, and token counts up to 64;
the other few-token shapes (M up to 128) go to the tiled kernel and are checked
alongside.  Reference: the oracle's fp64 GEMM of its own
quantisation, under the usual acceptance rule; the epilogue options against the
oracle as in the epilogue tests."""
import numpy as np
import pytest
import torch

import oracle
from fp8_dynamic_scaled_b200 import inputs
from gpu_util import assert_gemm_close, to_dev_bf16, to_host_u16

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
import fp8_dynamic_scaled_b200.binding as fp8  # noqa: E402
from test_gpu_epilogue import check_epilogue  # noqa: E402
from test_gpu_gemm import check_full, full_size_check, quantize_host, rand_bf16  # noqa: E402

E4M3, E5M2 = fp8.FP8_E4M3, fp8.FP8_E5M2
T, R = fp8.FP8_SCALE_TENSOR, fp8.FP8_SCALE_ROW


@pytest.mark.parametrize("M", [1, 2, 16, 33, 64, 100, 128])
@pytest.mark.parametrize("N,K", [(16, 128), (200, 512), (2368, 256), (3000, 640), (40000, 128), (20000, 1152),
                                 (300, 1040), (1000, 16)])
def test_decode_shapes_row_scales(M, N, K):
    x = rand_bf16((M, K), seed=M * 11 + K, lognormal_rows=True)
    w = rand_bf16((N, K), seed=N + K, std=0.02, lognormal_rows=True)
    check_full(x, w, R, R, what=f"decode {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(1, 264, 128), (64, 1000, 512)])
@pytest.mark.parametrize("am,bm", [(T, T), (T, R), (R, T)])
def test_decode_mixed_scale_modes(M, N, K, am, bm):
    x = rand_bf16((M, K), seed=M + 3, lognormal_rows=True)
    w = rand_bf16((N, K), seed=N + 5, std=0.02)
    check_full(x, w, am, bm, what=f"decode modes {am}/{bm}")


@pytest.mark.parametrize("fa,fb", [(E5M2, E5M2), (E4M3, E5M2), (E5M2, E4M3)])
def test_decode_e5m2_operands(fa, fb):
    x = rand_bf16((24, 768), seed=31, lognormal_rows=True)
    w = rand_bf16((1500, 768), seed=32, std=0.02)
    check_full(x, w, R, R, fa=fa, fb=fb, what=f"decode formats {fa}/{fb}")


def test_decode_output_row_stride():
    x = rand_bf16((40, 512), seed=41)
    w = rand_bf16((600, 512), seed=42, std=0.02)
    check_full(x, w, R, R, what="decode ldy", ldy=600 + 24)
    check_full(x, w, R, R, what="decode odd ldy", ldy=603)


@pytest.mark.parametrize("M,N,K", [(16, 2368, 512), (5, 4000, 256), (64, 3000, 640), (128, 520, 1024)])
def test_decode_epilogue_options(M, N, K):
    x = rand_bf16((M, K), seed=M * 7 + 1, lognormal_rows=True)
    w = rand_bf16((N, K), seed=N * 7 + 2, std=0.02)
    check_epilogue(x, w, R, R, seed=M, what=f"decode epilogue {M}x{N}x{K}")


@pytest.mark.parametrize("x_mode,w_mode", [(T, T), (R, R)])
@pytest.mark.parametrize("M", [1, 8, 128])
def test_decode_linear_forward(M, x_mode, w_mode):
    N, K = 3000, 1024
    x = rand_bf16((M, K), seed=51 + M, lognormal_rows=True)
    w = rand_bf16((N, K), seed=52, std=0.02)
    qb, sb = quantize_host(w, E4M3, w_mode)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = fp8.workspace_for(2, M, N, K, x_mode)
    fp8.fp8_linear_forward(to_dev_bf16(x), E4M3, x_mode, torch.from_numpy(qb).cuda(), torch.from_numpy(sb).cuda(),
                           w_mode, E4M3, y, ws)
    torch.cuda.synchronize()
    qa, sa = quantize_host(x, E4M3, x_mode)
    y_ref, bound = oracle.gemm_ref_full(qa, sa, x_mode, E4M3, qb, sb, w_mode, E4M3)
    assert_gemm_close(to_host_u16(y), y_ref, bound, f"decode linear M={M}")


@pytest.mark.parametrize("M", [1, 16, 64, 128])
def test_decode_llama70b_layer_full_size(M):
    """M tokens of the 28672 x 8192 layer: the whole W is streamed by every call."""
    x, w = inputs.llama70b_prefill(M=M)
    full_size_check(x, w, R, R, f"decode llama70b M={M}", npts=4000)
