// testing.cu -- device side of the testing entry points in include/fp8_testing.h.
//
// encode_f32_range_kernel puts the fp32 values whose bit patterns are first, first + 1,
// ..., first + n - 1 through the library's encode step, cvt_pair (round to nearest
// even, saturating to +-F_max), the same helper every quantize kernel applies to x / s
// ([FFS] "Scale 怎样把 Tensor 塞进 E4M3": X_fp8 = cast(clip(X / s))).  The values are
// generated from their index, so a test can sweep every fp32 pattern of a range
// without holding them in memory.
#include "common.cuh"
#include "kernels.h"

namespace fp8b {

template <int FMT>
__global__ void encode_f32_range_kernel(uint32_t first, int64_t n, uint8_t* __restrict__ q) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x * 2;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 2; i < n; i += stride) {
        const bool two = i + 1 < n;
        const float a = __uint_as_float(first + (uint32_t)i);
        const float b = two ? __uint_as_float(first + (uint32_t)(i + 1)) : 0.0f;
        const uint32_t c = cvt_pair<FMT>(a, b);
        q[i] = (uint8_t)(c & 0xFFu);
        if (two) q[i + 1] = (uint8_t)((c >> 8) & 0xFFu);
    }
}

cudaError_t launch_encode_f32_range(uint32_t first, int64_t n, int32_t fmt, uint8_t* q, cudaStream_t st) {
    const int threads = 256;
    const int64_t want = (n + 2 * threads - 1) / (2 * threads);
    const int grid = (int)(want < 148 * 16 ? want : 148 * 16);
    if (fmt == FP8_E4M3)
        encode_f32_range_kernel<FP8_E4M3><<<grid, threads, 0, st>>>(first, n, q);
    else
        encode_f32_range_kernel<FP8_E5M2><<<grid, threads, 0, st>>>(first, n, q);
    return cudaGetLastError();
}

}  // namespace fp8b
