"""The FP8 communication layer on the GPU path: libfp8's kernels under a one-rank
NCCL process group (one GPU is all a test box has).  Checks that the split
per-tensor scaling with the amax all-reduce equals fp8_quantize(TENSOR) bit for bit,
that the global amax equals the oracle's, and that the FP8 gathers return the
operand layout fp8_scaled_gemm consumes (the two-rank exchange itself is covered on
CPU by test_comm_gloo)."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from fp8_dynamic_scaled_b200 import inputs
from gpu_util import to_dev_bf16, to_host_u16

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
import fp8_dynamic_scaled_b200.binding as fp8  # noqa: E402
from fp8_dynamic_scaled_b200 import comm  # noqa: E402


@pytest.fixture(scope="module")
def nccl_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("fmt", [fp8.FP8_E4M3, fp8.FP8_E5M2])
def test_sharded_tensor_scaling_equals_tensor_mode(nccl_group, fmt):
    x_h = inputs.quant_sweep(rows=2048, cols=4096)
    x = to_dev_bf16(x_h)
    a = comm.global_amax(x)
    assert float(a.item()) == oracle.amax(x_h)
    q, s = comm.quantize_tensor_sharded(x, fmt)
    q2, s2, _ = fp8.empty_quant_outputs(2048, 4096, fp8.FP8_SCALE_TENSOR)
    fp8.fp8_quantize(x, fmt, fp8.FP8_SCALE_TENSOR, q2, s2, workspace=fp8.workspace_for(0, 2048, 0, 4096, 0))
    torch.cuda.synchronize()
    assert s.item() == s2.item() and torch.equal(q, q2)
    q_ref, s_ref, _ = oracle.quantize(x_h, fmt, oracle.TENSOR, dequant=False)
    assert np.float32(s.item()) == s_ref[0] and np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("mode", [comm.FP8_SCALE_TENSOR, comm.FP8_SCALE_ROW])
def test_all_gather_fp8_feeds_the_gemm(nccl_group, mode):
    g = np.random.default_rng(3)
    x_h = inputs.bf16_bits(g.standard_normal((256, 1024)).astype(np.float32))
    w_h = inputs.bf16_bits((g.standard_normal((512, 1024)) * 0.02).astype(np.float32))
    qx, sx = comm.all_gather_fp8(to_dev_bf16(x_h), fp8.FP8_E4M3, mode)
    qw, sw, _ = oracle.quantize(w_h, oracle.E4M3, oracle.ROW, dequant=False)
    y = torch.empty((256, 512), dtype=torch.bfloat16, device="cuda")
    fp8.fp8_scaled_gemm(qx, sx, mode, fp8.FP8_E4M3, torch.from_numpy(qw).cuda(), torch.from_numpy(sw).cuda(),
                        fp8.FP8_SCALE_ROW, fp8.FP8_E4M3, y)
    torch.cuda.synchronize()
    q_ref, s_ref, _ = oracle.quantize(x_h, oracle.E4M3, mode, dequant=False)
    assert np.array_equal(qx.cpu().numpy(), q_ref) and np.array_equal(sx.cpu().numpy(), s_ref)
    y_ref, bound = oracle.gemm_ref_full(q_ref, s_ref, mode, oracle.E4M3, qw, sw, oracle.ROW, oracle.E4M3)
    ok, _, _ = oracle.gemm_within_tolerance((to_host_u16(y).astype(np.uint32) << 16).view(np.float32), y_ref, bound)
    assert ok.all()
