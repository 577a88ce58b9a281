"""Build libfp8.so (the sm_100a kernels and the C ABI) in-tree with nvcc.

    python -m fp8_dynamic_scaled_b200.build [--verbose-ptxas]

No fast-math: fp32 division stays IEEE round-to-nearest and subnormals are kept,
which the bit-exact quantisation contract relies on.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfp8.so")
SOURCES = ["api.cu", "quantize.cu", "gemm_sm100.cu", "decode_sm100.cu", "wo_sm100.cu", "noalloc.cu", "testing.cu"]
HEADERS = ["common.cuh", "gemm_common.cuh", "kernels.h", "ptx.cuh"]
PUBLIC_HEADERS = [os.path.join(os.path.dirname(HERE), "include", h) for h in ("fp8.h", "fp8_testing.h")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + PUBLIC_HEADERS
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
           "-o", tmp] + [os.path.join(CSRC, s) for s in SOURCES]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
