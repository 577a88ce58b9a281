// kernels.h -- internal launcher interface between the C ABI (api.cu) and the
// kernels (quantize.cu, gemm_sm100.cu).  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

namespace fp8b {

struct QuantArgs {
    const uint16_t* x;
    int64_t rows, cols, ld;
    int32_t fmt, mode;
    uint8_t* q;
    void* scale;
    uint16_t* deq;          // nullable
    int32_t* status;        // nullable
    uint32_t* partials;     // per-tensor workspace (amax_partials_count() entries)
    // delayed scaling (hist_ring == nullptr otherwise)
    float* hist_ring;
    int32_t hist_len;
    int64_t hist_step;
    float* hist_pending;
    uint32_t* hist_ticket;
    // per-tensor cast with a caller's amax (launch_quantize_given)
    const float* amax_in;
};

int32_t amax_partials_count();
// The per-tensor workspace (fp8_workspace_size for TENSOR / DELAYED): the u32 partial
// maxima of the two-pass kernels, then the single-launch kernel's call counter and
// its per-CTA slots (8-byte words).
constexpr size_t kPartialsBytes = 4864;              // 4 * 1184 rounded up to 256
constexpr size_t kEpochOffset = kPartialsBytes;
constexpr size_t kSlotsOffset = kEpochOffset + 256;
constexpr size_t kTensorWorkspaceBytes = kSlotsOffset + 8 * 1184;
cudaError_t launch_quantize_tensor(const QuantArgs& a, cudaStream_t st);
cudaError_t launch_quantize_grouped(const QuantArgs& a, cudaStream_t st);
cudaError_t launch_fill_scale(float* s, int64_t n, float v, cudaStream_t st);
cudaError_t launch_amax(const QuantArgs& a, float* out, cudaStream_t st);
cudaError_t launch_quantize_given(const QuantArgs& a, cudaStream_t st);

struct GemmArgs {
    const uint8_t* a;        // [M, K] codes
    const uint8_t* b;        // [N, K] codes
    const void* sa;
    const void* sb;
    int32_t a_mode, b_mode;  // TENSOR/ROW (any mix), BLOCK pair, or MX32 pair
    int32_t fmt_a, fmt_b;
    int64_t M, N, K;
    uint16_t* y;             // bf16 [M, N], row stride ldy (null: FP8 output only)
    int64_t ldy;
    int32_t* status;
    // epilogue options (all null: plain bf16 output)
    const uint16_t* bias;    // bf16 [N]
    float* amax;             // running max |y|
    uint8_t* yq;             // FP8 codes [M, ldq]
    const float* yq_scale;   // s_y
    int32_t yq_fmt;
    int64_t ldq;
    // the kernel just before the GEMM on the stream wrote A and its scales and nothing
    // else: the GEMM may start on B before A is ready (programmatic dependent launch)
    bool a_from_previous_kernel;
};

cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t st);

// Limit of every pipeline wait (and of the per-tensor kernel's grid-wide exchange) in
// the kernels launched from now on (0: the default, 4 s); only the testing entry point
// fp8_testing_set_wait_limit_ns sets it.  wait_limit_ns() is read when a launch is
// prepared.
void set_wait_limit_ns(uint64_t ns);
uint64_t wait_limit_ns();

// testing.cu: the n fp32 values with bit patterns first .. first + n - 1 through the
// encode step of the quantize kernels (n >= 1, first + n <= 2^32, q holds n bytes).
cudaError_t launch_encode_f32_range(uint32_t first, int64_t n, int32_t fmt, uint8_t* q, cudaStream_t st);

struct WoArgs {              // weight-only FP8 linear (wo_sm100.cu)
    const uint16_t* x;       // bf16 [M, K], row stride ldx
    int64_t ldx;
    const uint8_t* w;        // FP8 codes [N, K]
    const void* sw;          // fp32 scale: [1] or [N]
    bool w_row_scales;
    int32_t w_fmt;
    int64_t M, N, K;
    uint16_t* y;             // bf16 [M, N], row stride ldy
    int64_t ldy;
    int32_t* status;
};
cudaError_t launch_weight_only(const WoArgs& g, cudaStream_t st);
cudaError_t launch_zero_output(uint16_t* y, int64_t M, int64_t N, int64_t ldy, cudaStream_t st);
cudaError_t launch_zero_k_epilogue(const GemmArgs& g, cudaStream_t st);

}  // namespace fp8b
