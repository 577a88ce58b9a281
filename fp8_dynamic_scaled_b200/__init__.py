"""fp8_dynamic_scaled_b200 -- the FP8 runtime linear path on B200 (sm_100a).

    X --amax--> s = amax / F_max --clip, RNE cast--> X_fp8;  Y = s_x s_w (X_fp8 W_fp8^T) in BF16

The work happens in libfp8.so (hand-written CUDA: fused quantize kernels and a
tcgen05/TMEM/TMA FP8 GEMM), whose C ABI is include/fp8.h.  The names exported
here (fp8_quantize, fp8_scaled_gemm, fp8_linear_forward, ...) are the ctypes
binding of that ABI and are loaded on first use; ``inputs`` holds the seeded
synthetic workload generators.
"""
from __future__ import annotations

import importlib

__all__ = ["fp8_abi_version", "fp8_status_string", "fp8_device_check", "fp8_workspace_size", "fp8_quantize",
           "fp8_scaled_gemm", "fp8_linear_forward", "fp8_amax", "fp8_quantize_with_amax", "fp8_scaled_gemm_ex",
           "fp8_linear_forward_ex", "fp8_weight_only_linear", "History", "FP8Error", "binding", "inputs"]


def __getattr__(name):
    if name == "inputs":
        return importlib.import_module(".inputs", __name__)
    binding = importlib.import_module(".binding", __name__)
    if name == "binding":
        return binding
    if hasattr(binding, name):
        return getattr(binding, name)
    raise AttributeError(name)
