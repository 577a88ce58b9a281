"""Quantize tensors with more than 2^31 elements.

262,145 rows of 8,192 bf16 values (2,147,491,840 elements, 4.3 GB) go through the
per-tensor path (the single-launch kernel: element and vector offsets past 32 bits) and
the per-row path (262,145 CTAs of the row kernel).  Codes and scales are compared byte
for byte with the oracle.  The input is drawn on the device from a seeded generator and
copied to the host once for the oracle."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
import fp8_dynamic_scaled_b200.binding as fp8  # noqa: E402

ROWS, COLS = 262_145, 8_192                       # ROWS * COLS > 2^31


@pytest.fixture(scope="module")
def big_input():
    g = torch.Generator(device="cuda")
    g.manual_seed(2031)
    x = torch.empty((ROWS, COLS), dtype=torch.bfloat16, device="cuda")
    for r0 in range(0, ROWS, 16384):            # row blocks: a spread of magnitudes
        r1 = min(ROWS, r0 + 16384)
        blk = torch.randn((r1 - r0, COLS), generator=g, device="cuda", dtype=torch.float32)
        blk *= torch.exp(torch.randn((r1 - r0, 1), generator=g, device="cuda"))
        x[r0:r1] = blk.to(torch.bfloat16)
    x[ROWS - 1, COLS - 1] = 3.0e4                 # the a_max sits in the last element
    x_host = x.view(torch.int16).cpu().numpy().view(np.uint16)
    yield x, x_host
    del x
    torch.cuda.empty_cache()


def test_per_tensor_beyond_2pow31_elements(big_input):
    x, x_host = big_input
    assert x.numel() > 2 ** 31
    q, s, _ = fp8.empty_quant_outputs(ROWS, COLS, fp8.FP8_SCALE_TENSOR)
    ws = fp8.workspace_for(0, ROWS, 0, COLS, fp8.FP8_SCALE_TENSOR)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8.fp8_quantize(x, fp8.FP8_E4M3, fp8.FP8_SCALE_TENSOR, q, s, dev_status=st, workspace=ws)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rq, rs, _ = oracle.quantize(x_host, fp8.FP8_E4M3, oracle.TENSOR, dequant=False)
    assert s.cpu().numpy().view(np.uint32)[0] == rs.view(np.uint32)[0]
    got = q.cpu().numpy()
    del q
    assert np.array_equal(got.reshape(-1), rq.reshape(-1))


def test_per_row_beyond_2pow31_elements(big_input):
    x, x_host = big_input
    q, s, _ = fp8.empty_quant_outputs(ROWS, COLS, fp8.FP8_SCALE_ROW)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8.fp8_quantize(x, fp8.FP8_E4M3, fp8.FP8_SCALE_ROW, q, s, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rq, rs, _ = oracle.quantize(x_host, fp8.FP8_E4M3, oracle.ROW, dequant=False)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32).reshape(-1))
    got = q.cpu().numpy()
    del q
    assert np.array_equal(got.reshape(-1), rq.reshape(-1))


def test_gemm_output_beyond_2pow31_elements():
    """Y [65536, 32768] (2^31 outputs, 4.3 GB of bf16) from the CTA-pair kernel with
    per-row scales, K = 256; 8,192 sampled outputs, the last rows and columns among them,
    against the oracle under the acceptance rule."""
    M, N, K = 65536, 32768, 256
    g = np.random.default_rng(91)
    qa = g.integers(0, 0x7E, (M, K), dtype=np.uint8) | (g.integers(0, 2, (M, K), dtype=np.uint8) << 7)
    qb = g.integers(0, 0x7E, (N, K), dtype=np.uint8) | (g.integers(0, 2, (N, K), dtype=np.uint8) << 7)
    sa = np.exp(g.standard_normal(M)).astype(np.float32) * np.float32(1e-3)
    sb = np.exp(g.standard_normal(N)).astype(np.float32) * np.float32(1e-3)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8.fp8_scaled_gemm(torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda(), fp8.FP8_SCALE_ROW, fp8.FP8_E4M3,
                        torch.from_numpy(qb).cuda(), torch.from_numpy(sb).cuda(), fp8.FP8_SCALE_ROW, fp8.FP8_E4M3,
                        y, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    pm = np.concatenate([g.integers(0, M, 8000), np.full(96, M - 1), np.arange(M - 96, M)])
    pn = np.concatenate([g.integers(0, N, 8000), np.arange(N - 96, N), np.full(96, N - 1)])
    yv = y[torch.from_numpy(pm).cuda(), torch.from_numpy(pn).cuda()].float().cpu().numpy().astype(np.float64)
    del y
    torch.cuda.empty_cache()
    y_ref, bound = oracle.gemm_ref_points(qa, sa, oracle.ROW, fp8.FP8_E4M3, qb, sb, oracle.ROW, fp8.FP8_E4M3, pm, pn)
    ok, err, _ = oracle.gemm_within_tolerance(yv, y_ref, bound)
    assert ok.all(), f"{int((~ok).sum())} sampled outputs off the oracle (max err {err.max():.3g})"
