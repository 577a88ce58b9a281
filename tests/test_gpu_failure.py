"""Failure path of the bounded waits, without faulting or hanging the GPU.

Every mbarrier wait in the GEMM kernels is bounded in time.  A testing entry point
(include/fp8_testing.h) shortens the limit to 1 microsecond, and each kernel is given
a K deep enough (65,536) that its pipeline takes far longer than that, so a wait runs
out: the kernel must report FP8_ERR_TIMEOUT in dev_status, drain the copies and MMAs it
has issued, free its tensor memory and exit.  The same device must then run the same
call at the default limit with a correct result (checked against the oracle)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_gemm_close, to_host_u16

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
import fp8_dynamic_scaled_b200.binding as fp8  # noqa: E402

E4M3, T, R = fp8.FP8_E4M3, fp8.FP8_SCALE_TENSOR, fp8.FP8_SCALE_ROW
DEEP_K = 65536
SHORT_LIMIT_NS = 1000


def _operands(M, N, K, seed):
    """Small-integer codes (exact products) with per-row scales."""
    g = np.random.default_rng(seed)
    qa = oracle.encode(g.integers(-3, 4, (M, K)).astype(np.float32), E4M3).reshape(M, K)
    qb = oracle.encode(g.integers(-3, 4, (N, K)).astype(np.float32), E4M3).reshape(N, K)
    sa = (1.0 + g.random(M)).astype(np.float32) / 64
    sb = (1.0 + g.random(N)).astype(np.float32) / 64
    return qa, sa, qb, sb


def _run(kind, qa, sa, qb, sb, M, N, status):
    a, b = torch.from_numpy(qa).cuda(), torch.from_numpy(qb).cuda()
    sa_d, sb_d = torch.from_numpy(sa).cuda(), torch.from_numpy(sb).cuda()
    y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    if kind == "weight_only":
        x = (a.view(torch.float8_e4m3fn).float() * sa_d[:, None]).to(torch.bfloat16)
        fp8.fp8_weight_only_linear(x, b, sb_d, R, E4M3, y, dev_status=status)
    else:
        fp8.fp8_scaled_gemm(a, sa_d, R, E4M3, b, sb_d, R, E4M3, y, dev_status=status)
    torch.cuda.synchronize()
    return y


# M picks the kernel: 256 -> CTA pair, 128 -> single-CTA tiles, 16 -> weight-streaming
# decode kernel; weight-only at 8 tokens -> the BF16 tensor-core kernel
@pytest.mark.parametrize("kind,M,N", [("tiled", 128, 256), ("pair", 256, 256), ("decode", 16, 256),
                                      ("weight_only", 8, 256)])
def test_bounded_wait_runs_out_then_device_recovers(kind, M, N):
    qa, sa, qb, sb = _operands(M, N, DEEP_K, seed=M + N)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8.fp8_testing_set_wait_limit_ns(SHORT_LIMIT_NS)
    try:
        _run(kind, qa, sa, qb, sb, M, N, status)
    finally:
        fp8.fp8_testing_set_wait_limit_ns(0)
    assert int(status.item()) == fp8.FP8_ERR_TIMEOUT, f"{kind}: status {int(status.item())}"
    # the context is intact: the same kernel at the default limit is correct
    qa, sa, qb, sb = _operands(M, N, 1024, seed=M + N + 1)
    status.zero_()
    y = _run(kind, qa, sa, qb, sb, M, N, status)
    assert int(status.item()) == 0
    if kind == "weight_only":
        x_bits = to_host_u16((torch.from_numpy(qa).cuda().view(torch.float8_e4m3fn).float()
                              * torch.from_numpy(sa).cuda()[:, None]).to(torch.bfloat16))
        y_ref, bound = oracle.weight_only_ref(x_bits, qb, sb, oracle.ROW, oracle.E4M3)
    else:
        y_ref, bound = oracle.gemm_ref_full(qa, sa, oracle.ROW, oracle.E4M3, qb, sb, oracle.ROW, oracle.E4M3)
    assert_gemm_close(to_host_u16(y), y_ref, bound, f"{kind} after the timeout")


def test_small_gemm_after_a_timeout():
    """The 128 x 256 x 256 per-tensor GEMM right after a timed-out launch."""
    qa, sa, qb, sb = _operands(128, 256, DEEP_K, seed=3)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8.fp8_testing_set_wait_limit_ns(SHORT_LIMIT_NS)
    try:
        _run("tiled", qa, sa, qb, sb, 128, 256, status)
    finally:
        fp8.fp8_testing_set_wait_limit_ns(0)
    assert int(status.item()) == fp8.FP8_ERR_TIMEOUT
    qa, sa, qb, sb = _operands(128, 256, 256, seed=4)
    status.zero_()
    y = _run("tiled", qa, sa, qb, sb, 128, 256, status)
    assert int(status.item()) == 0
    y_ref, bound = oracle.gemm_ref_full(qa, sa, oracle.ROW, oracle.E4M3, qb, sb, oracle.ROW, oracle.E4M3)
    assert_gemm_close(to_host_u16(y), y_ref, bound, "128x256x256 after the timeout")
