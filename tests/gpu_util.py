"""Helpers shared by the GPU parity tests: numpy <-> torch transfers of bf16 bit
patterns and the standard tolerance check.  Holds none of the method's arithmetic."""
import numpy as np
import torch

import oracle


def to_dev_bf16(u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).cuda()


def to_host_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_bits_to_f64(u16: np.ndarray) -> np.ndarray:
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_gemm_close(y_gpu_u16: np.ndarray, y_ref: np.ndarray, bound: np.ndarray, what: str):
    y = bf16_bits_to_f64(y_gpu_u16)
    ok, err, lim = oracle.gemm_within_tolerance(y, y_ref, bound)
    if not ok.all():
        idx = np.argwhere(~ok)[:8]
        detail = [(tuple(int(v) for v in i), float(y[tuple(i)]), float(y_ref[tuple(i)]), float(lim[tuple(i)]))
                  for i in idx]
        raise AssertionError(f"{what}: {int((~ok).sum())} of {ok.size} outputs out of tolerance; first {detail}")


def first_mismatch(a: np.ndarray, b: np.ndarray):
    bad = np.argwhere(a != b)
    if bad.size == 0:
        return None
    i = tuple(int(v) for v in bad[0])
    return i, a[i], b[i], int(bad.shape[0])
