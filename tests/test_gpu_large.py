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
