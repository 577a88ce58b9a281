"""fp8_linear_forward_noalloc: the linear forward for callers that cannot allocate.

Such callers (plug-ins of a host program that owns all device memory, or code that
must not call cudaMalloc because it may synchronise the device) get no workspace
argument; the scratch is a fixed device array inside libfp8.so.  These tests call
the entry point through the C ABI, two calls in a row, and require its output to be
bit-identical to fp8_linear_forward's (the entry point that takes a caller
workspace; both run the same kernels on the same inputs) and within the GEMM
acceptance rule of the oracle's fp64 reference.  The file is named so that pytest
collects it last; it does not depend on the tests before it."""
import numpy as np
import pytest
import torch

import oracle
from fp8_dynamic_scaled_b200 import inputs
from gpu_util import to_dev_bf16, to_host_u16

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
import fp8_dynamic_scaled_b200.binding as fp8  # noqa: E402

E4M3 = fp8.FP8_E4M3


def _operands(M, N, K, seed, w_mode):
    g = np.random.default_rng(seed)
    x = inputs.bf16_bits(g.standard_normal((M, K)).astype(np.float32)
                         * np.exp(g.standard_normal((M, 1))).astype(np.float32))
    w = inputs.bf16_bits((g.standard_normal((N, K)) * 0.02).astype(np.float32))
    wq, ws, _ = oracle.quantize(w, oracle.E4M3, w_mode, dequant=False)
    return x, torch.from_numpy(wq).cuda(), torch.from_numpy(np.ascontiguousarray(ws)).cuda()


def _against_oracle(y_u16, x_u16, wq, ws, x_mode, w_mode):
    """|y - y_ref| <= 1e-3 * sum_k|terms| + 1 bf16 ulp(y_ref), y_ref the oracle's fp64 GEMM of
    the oracle's own quantisation of X and the given weight codes."""
    qa, sa, _ = oracle.quantize(x_u16, oracle.E4M3, x_mode, dequant=False)
    y_ref, bound = oracle.gemm_ref_full(qa, sa, x_mode, oracle.E4M3, wq.cpu().numpy(), ws.cpu().numpy(), w_mode,
                                        oracle.E4M3)
    y = (y_u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ok, err, lim = oracle.gemm_within_tolerance(y, y_ref, bound)
    assert ok.all(), f"{int((~ok).sum())} outputs off the oracle beyond the rule (max err {err.max():.3g})"


@pytest.mark.parametrize("x_mode,w_mode", [(fp8.FP8_SCALE_TENSOR, fp8.FP8_SCALE_TENSOR),
                                           (fp8.FP8_SCALE_ROW, fp8.FP8_SCALE_ROW),
                                           (fp8.FP8_SCALE_BLOCK_1x128, fp8.FP8_SCALE_BLOCK_128x128),
                                           (fp8.FP8_SCALE_MX32, fp8.FP8_SCALE_MX32)])
def test_noalloc_matches_workspace_entry_point_twice(x_mode, w_mode):
    M, N, K = 200, 384, 1024
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call, seed in enumerate((1, 2)):        # two calls in a row; the second sees the first's leftovers
        x_h, wq, ws = _operands(M, N, K, seed + 10 * x_mode, w_mode)
        x = to_dev_bf16(x_h)
        y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        fp8.fp8_linear_forward(x, E4M3, x_mode, wq, ws, w_mode, E4M3, y_ref, fp8.workspace_for(2, M, N, K, x_mode),
                               dev_status=status)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        fp8.fp8_linear_forward_noalloc(x, E4M3, x_mode, wq, ws, w_mode, E4M3, y, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), \
            f"call {call}: the no-allocation entry point differs from fp8_linear_forward"
        _against_oracle(to_host_u16(y), x_h, wq, ws, x_mode, w_mode)


def test_noalloc_delayed_history_two_steps():
    M, N, K = 256, 256, 512
    _, wq, ws = _operands(M, N, K, 5, fp8.FP8_SCALE_TENSOR)
    h_ref, h_new = fp8.History(16), fp8.History(16)
    ring = np.zeros(16, np.float32)
    ws_lin = fp8.workspace_for(2, M, N, K, fp8.FP8_SCALE_DELAYED)
    for t in range(2):
        x_h = inputs.delayed_step_input(t, M=M, K=K)
        x = to_dev_bf16(x_h)
        y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        fp8.fp8_linear_forward(x, E4M3, fp8.FP8_SCALE_DELAYED, wq, ws, fp8.FP8_SCALE_TENSOR, E4M3, y_ref, ws_lin,
                               hist=h_ref)
        fp8.fp8_linear_forward_noalloc(x, E4M3, fp8.FP8_SCALE_DELAYED, wq, ws, fp8.FP8_SCALE_TENSOR, E4M3, y,
                                       hist=h_new)
        torch.cuda.synchronize()
        assert torch.equal(h_ref.ring, h_new.ring) and h_new.step == t + 1
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), f"step {t}: outputs differ"
        qa, s_t, _, _ = oracle.delayed_step(x_h, oracle.E4M3, ring, t)
        assert np.array_equal(h_new.ring.cpu().numpy().view(np.uint32), ring.view(np.uint32)), f"step {t} ring"
        y_o, bound = oracle.gemm_ref_full(qa, np.array([s_t], np.float32), oracle.TENSOR, oracle.E4M3,
                                          wq.cpu().numpy(), ws.cpu().numpy(), oracle.TENSOR, oracle.E4M3)
        a = (to_host_u16(y).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        ok, err, _ = oracle.gemm_within_tolerance(a, y_o, bound)
        assert ok.all(), f"step {t}: {int((~ok).sum())} outputs off the oracle beyond the rule"


def test_noalloc_rejects_inputs_beyond_its_scratch():
    M, K, N = 1024, 8192, 256           # 8 MiB of activation codes > the 4 MiB scratch
    assert fp8.fp8_workspace_size(2, M, N, K, fp8.FP8_SCALE_ROW) > fp8.FP8_NOALLOC_SCRATCH_BYTES
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    s = torch.ones(N, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fp8.FP8Error) as e:
        fp8.fp8_linear_forward_noalloc(x, E4M3, fp8.FP8_SCALE_ROW, w, s, fp8.FP8_SCALE_ROW, E4M3, y)
    assert e.value.status == fp8.FP8_ERR_WORKSPACE
