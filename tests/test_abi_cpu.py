"""CPU-side checks of the C ABI: the library builds for sm_100a, loads, exports every
entry point include/fp8.h declares, and rejects bad arguments before touching a
device.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from fp8_dynamic_scaled_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def declared_symbols():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"FP8_API\s+[\w\s\*]+?\b(fp8_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), f"{n} not exported"
    from fp8_dynamic_scaled_b200 import binding
    assert set(binding.EXPORTED) <= set(names)


def test_version_and_status_strings(lib):
    from fp8_dynamic_scaled_b200 import binding as b
    assert b.fp8_abi_version() == 2
    assert b.fp8_status_string(0) == "FP8_OK"
    assert b.fp8_status_string(5) == "FP8_ERR_TIMEOUT"
    assert b.fp8_status_string(99) == "FP8_ERR_UNKNOWN"


def test_workspace_sizes():
    from fp8_dynamic_scaled_b200 import binding as b
    assert b.fp8_workspace_size(0, 128, 0, 256, b.FP8_SCALE_TENSOR) >= 4 * 148 * 8
    assert b.fp8_workspace_size(0, 128, 0, 256, b.FP8_SCALE_ROW) == 0
    assert b.fp8_workspace_size(1, 128, 256, 256, b.FP8_SCALE_ROW) == 0
    n = b.fp8_workspace_size(2, 4096, 28672, 8192, b.FP8_SCALE_ROW)
    assert n >= 4096 * 8192 + 4 * 4096
    assert b.fp8_workspace_size(2, 4096, 8192, 8192, b.FP8_SCALE_MX32) >= 4096 * 8192 + 4096 * 256


def test_argument_validation_without_device(lib):
    """Invalid arguments are refused synchronously, before any CUDA call."""
    from fp8_dynamic_scaled_b200 import binding as b
    L = b._lib
    P = 0x1000  # a 16-byte aligned fake device address; never dereferenced on these paths
    # cols % 16 != 0
    assert L.fp8_quantize(P, 4, 24, 24, 0, 1, P, P, None, None, None, None, 0, None) == b.FP8_ERR_INVALID_ARG
    # unknown format / mode
    assert L.fp8_quantize(P, 4, 32, 32, 7, 1, P, P, None, None, None, None, 0, None) == b.FP8_ERR_INVALID_ARG
    assert L.fp8_quantize(P, 4, 32, 32, 0, 9, P, P, None, None, None, None, 0, None) == b.FP8_ERR_INVALID_ARG
    # MX32 needs E4M3
    assert L.fp8_quantize(P, 4, 32, 32, 1, 4, P, P, None, None, None, None, 0, None) == b.FP8_ERR_INVALID_ARG
    # DELAYED needs a history
    assert L.fp8_quantize(P, 4, 32, 32, 0, 5, P, P, None, None, None, None, 0, None) == b.FP8_ERR_INVALID_ARG
    # misaligned x and ld
    assert L.fp8_quantize(P + 2, 4, 32, 32, 0, 1, P, P, None, None, None, None, 0, None) == b.FP8_ERR_ALIGNMENT
    assert L.fp8_quantize(P, 4, 32, 36, 0, 1, P, P, None, None, None, None, 0, None) == b.FP8_ERR_ALIGNMENT
    # GEMM: K % 16, unsupported mode pair, ldy
    assert L.fp8_scaled_gemm(P, P, 1, 0, P, P, 1, 0, 16, 16, 24, P, 16, None, None, 0, None) == b.FP8_ERR_INVALID_ARG
    assert L.fp8_scaled_gemm(P, P, 2, 0, P, P, 1, 0, 16, 16, 32, P, 16, None, None, 0, None) == b.FP8_ERR_INVALID_ARG
    assert L.fp8_scaled_gemm(P, P, 4, 0, P, P, 4, 1, 16, 16, 32, P, 16, None, None, 0, None) == b.FP8_ERR_INVALID_ARG
    assert L.fp8_scaled_gemm(P, P, 1, 0, P, P, 1, 0, 16, 16, 32, P, 12, None, None, 0, None) == b.FP8_ERR_INVALID_ARG
    assert L.fp8_scaled_gemm(P, P, 1, 0, P, P, 1, 0, 16, 16, 32, P + 1, 20, None, None, 0, None) == b.FP8_ERR_ALIGNMENT
    # linear forward: workspace missing / too small
    assert L.fp8_linear_forward(P, 16, 32, 32, 0, 1, None, P, P, 1, 0, 16, P, 16, None, None, 0, None) \
        == b.FP8_ERR_WORKSPACE
    assert L.fp8_linear_forward(P, 16, 32, 32, 0, 3, None, P, P, 1, 0, 16, P, 16, None, P, 1 << 20, None) \
        == b.FP8_ERR_INVALID_ARG


def test_product_code_never_imports_the_oracle():
    """The CUDA path and the oracle share nothing: no product source mentions it."""
    pkg = os.path.join(ROOT, "fp8_dynamic_scaled_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn), encoding="utf-8").read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "fp8_oracle" not in text and "liboracle" not in text, fn
