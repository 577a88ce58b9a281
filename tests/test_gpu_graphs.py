"""CUDA-graph capture and replay of the hot path.

Every call is asynchronous on the caller's stream and allocates nothing, so a CUDA graph
can hold it: captured once after a warm-up call (which fills the library's host-side
caches), then replayed with new data copied into the captured input buffer.  The
single-launch per-tensor quantize keeps a call counter in its workspace, so each replay
takes a new call number and its grid-wide amax exchange accepts only slots of its own
replay.  fp8_linear_forward launches its GEMM as the programmatic dependent of the X
quantize, an edge the graph keeps.  Every replay is compared with the oracle on its own
inputs: codes, scale and dequant bit for bit; GEMM outputs under the acceptance rule."""
import numpy as np
import pytest
import torch

import oracle
from fp8_dynamic_scaled_b200 import inputs
from gpu_util import first_mismatch, to_dev_bf16, to_host_u16

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
import fp8_dynamic_scaled_b200.binding as fp8  # noqa: E402

E4, T, R = fp8.FP8_E4M3, fp8.FP8_SCALE_TENSOR, fp8.FP8_SCALE_ROW


def _bf16(shape, seed, spread=1.0, std=1.0):
    g = np.random.default_rng(seed)
    x = g.standard_normal(shape).astype(np.float32) * np.float32(std)
    x *= np.exp(spread * g.standard_normal((shape[0], 1))).astype(np.float32)
    return inputs.bf16_bits(x)


def _capture(fn, stream):
    with torch.cuda.stream(stream):
        fn()                                      # warm-up: host-side caches
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
        fn()
    return g


def test_per_tensor_single_launch_replays():
    rows, cols = 2048, 8192                       # 16 Mi elements: the single-launch kernel
    xd = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda")
    xd.copy_(to_dev_bf16(_bf16((rows, cols), 1)))
    q, s, d = fp8.empty_quant_outputs(rows, cols, T, dequant=True)
    ws = fp8.workspace_for(0, rows, 0, cols, T)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.Stream()
    g = _capture(lambda: fp8.fp8_quantize(xd, E4, T, q, s, dequant=d, dev_status=st, workspace=ws, stream=stream),
                 stream)
    for i in range(4):
        x = _bf16((rows, cols), 10 + i, spread=0.5 * i)
        if i == 2:
            x[5, 7] = 0x4F00                      # a much larger amax than the replays before
        xd.copy_(to_dev_bf16(x))
        g.replay()
        torch.cuda.synchronize()
        assert int(st.item()) == 0, f"replay {i}: status {int(st.item())}"
        rq, rs, rd = oracle.quantize(x, E4, oracle.TENSOR, dequant=True)
        assert s.cpu().numpy().view(np.uint32)[0] == rs.view(np.uint32)[0], f"replay {i}: scale"
        assert first_mismatch(q.cpu().numpy(), rq) is None, f"replay {i}: codes"
        assert first_mismatch(to_host_u16(d), rd) is None, f"replay {i}: dequant"


@pytest.mark.parametrize("M", [16, 512])          # the decode kernel; the CTA-pair kernel
def test_linear_forward_replays(M):
    K, N = 1024, 2048
    w = _bf16((N, K), 2, spread=0.3, std=0.02)
    qw, sw, _ = oracle.quantize(w, E4, oracle.ROW, dequant=False)
    wq, wsd = torch.from_numpy(qw).cuda(), torch.from_numpy(np.ascontiguousarray(sw)).cuda()
    xd = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    xd.copy_(to_dev_bf16(_bf16((M, K), 3)))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    lws = fp8.workspace_for(2, M, N, K, R)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.Stream()
    g = _capture(lambda: fp8.fp8_linear_forward(xd, E4, R, wq, wsd, R, E4, y, lws, dev_status=st, stream=stream),
                 stream)
    for i in range(3):
        x = _bf16((M, K), 20 + i, spread=1.0)
        xd.copy_(to_dev_bf16(x))
        g.replay()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        qa, sa, _ = oracle.quantize(x, E4, oracle.ROW, dequant=False)
        y_ref, bound = oracle.gemm_ref_full(qa, sa, oracle.ROW, E4, qw, sw, oracle.ROW, E4)
        yv = (to_host_u16(y).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        ok, err, _ = oracle.gemm_within_tolerance(yv, y_ref, bound)
        assert ok.all(), f"M {M} replay {i}: {int((~ok).sum())} outputs off the oracle (max err {err.max():.3g})"
