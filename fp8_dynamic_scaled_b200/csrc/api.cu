// api.cu -- the C ABI of libfp8.so (declared in include/fp8.h): argument checks,
// device gate, workspace carving and kernel dispatch.  No compute happens here.
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "../../include/fp8_testing.h"

using namespace fp8b;

namespace {

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// The compute capability major the gate sees instead of the device's own, from the
// environment variable FP8_B200_FORCE_CC_MAJOR (read once per process), or -1: a test
// uses it to drive the unsupported-device path on a B200.
int forced_cc_major() {
    static const int v = [] {
        const char* e = std::getenv("FP8_B200_FORCE_CC_MAJOR");
        if (e == nullptr || *e == '\0') return -1;
        char* end = nullptr;
        const long n = std::strtol(e, &end, 10);
        return (end != e && *end == '\0' && n >= 0 && n < 100) ? (int)n : -1;
    }();
    return v;
}

// FP8_OK when the current device is compute capability 10.x.
int32_t device_gate() {
    static int cache[kMaxDevices];   // 0 unknown, 1 ok, 2 unsupported
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP8_ERR_CUDA;
    if (dev >= 0 && dev < kMaxDevices && cache[dev] != 0) return cache[dev] == 1 ? FP8_OK : FP8_ERR_UNSUPPORTED_DEVICE;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return FP8_ERR_CUDA;
    if (forced_cc_major() >= 0) major = forced_cc_major();
    const int ok = major == 10 ? 1 : 2;
    if (dev >= 0 && dev < kMaxDevices) cache[dev] = ok;
    return ok == 1 ? FP8_OK : FP8_ERR_UNSUPPORTED_DEVICE;
}

int64_t scale_bytes(int32_t mode, int64_t rows, int64_t cols) {
    switch (mode) {
    case FP8_SCALE_TENSOR:
    case FP8_SCALE_DELAYED: return 4;
    case FP8_SCALE_ROW: return 4 * rows;
    case FP8_SCALE_BLOCK_1x128: return 4 * rows * cdiv(cols, 128);
    case FP8_SCALE_BLOCK_128x128: return 4 * cdiv(rows, 128) * cdiv(cols, 128);
    case FP8_SCALE_MX32: return rows * (cols / 32);
    default: return -1;
    }
}

size_t partials_bytes() { return align_up(kTensorWorkspaceBytes, 256); }

int32_t cuda_status(cudaError_t e) { return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA; }

int32_t check_quantize_args(const void* x, int64_t rows, int64_t cols, int64_t ld, int32_t fmt, int32_t mode,
                            const uint8_t* q, const void* scale, const fp8_history_t* hist, const void* deq,
                            bool need_q = true) {
    if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (mode < FP8_SCALE_TENSOR || mode > FP8_SCALE_DELAYED) return FP8_ERR_INVALID_ARG;
    if (mode == FP8_SCALE_MX32 && fmt != FP8_E4M3) return FP8_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols) return FP8_ERR_INVALID_ARG;
    if (rows >= ((int64_t)1 << 40) || cols >= ((int64_t)1 << 40)) return FP8_ERR_INVALID_ARG;
    if (cols % 16 != 0) return FP8_ERR_INVALID_ARG;
    if (mode == FP8_SCALE_MX32 && cols % 32 != 0) return FP8_ERR_INVALID_ARG;
    if (scale == nullptr && scale_bytes(mode, rows, cols) > 0) return FP8_ERR_INVALID_ARG;
    const bool empty = rows == 0 || cols == 0;
    if (!empty && (x == nullptr || (need_q && q == nullptr))) return FP8_ERR_INVALID_ARG;
    if (mode == FP8_SCALE_DELAYED) {
        if (!hist || !hist->ring_dev || !hist->pending_dev || !hist->ticket_dev || hist->len < 1 || hist->step < 0)
            return FP8_ERR_INVALID_ARG;
    }
    if (ld % 8 != 0) return FP8_ERR_ALIGNMENT;
    if (!aligned16(x) || !aligned16(q) || !aligned16(deq)) return FP8_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(scale) & (mode == FP8_SCALE_MX32 ? 0u : 3u)) != 0) return FP8_ERR_ALIGNMENT;
    return FP8_OK;
}

int32_t quantize_impl(const void* x, int64_t rows, int64_t cols, int64_t ld, int32_t fmt, int32_t mode, uint8_t* q,
                      void* scale, fp8_history_t* hist, void* deq, int32_t* status, void* ws, size_t ws_bytes,
                      cudaStream_t st) {
    QuantArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.fmt = fmt;
    a.mode = mode;
    a.q = q;
    a.scale = scale;
    a.deq = static_cast<uint16_t*>(deq);
    a.status = status;
    if (mode == FP8_SCALE_TENSOR || mode == FP8_SCALE_DELAYED) {
        if (ws == nullptr || ws_bytes < partials_bytes()) return FP8_ERR_WORKSPACE;
        if ((reinterpret_cast<uintptr_t>(ws) & 3u) != 0) return FP8_ERR_ALIGNMENT;
        a.partials = static_cast<uint32_t*>(ws);
        if (mode == FP8_SCALE_DELAYED) {
            a.hist_ring = hist->ring_dev;
            a.hist_len = hist->len;
            a.hist_step = hist->step;
            a.hist_pending = hist->pending_dev;
            a.hist_ticket = hist->ticket_dev;
        }
        int32_t rc = cuda_status(launch_quantize_tensor(a, st));
        if (rc == FP8_OK && mode == FP8_SCALE_DELAYED) hist->step += 1;
        return rc;
    }
    if (rows == 0 || cols == 0) {
        // amax of an empty group is 0: floor scales (MX: the zero byte) for the groups that exist
        const int64_t n = scale_bytes(mode, rows, cols) / (mode == FP8_SCALE_MX32 ? 1 : 4);
        if (mode == FP8_SCALE_MX32 || n == 0) return n == 0 ? FP8_OK : cuda_status(cudaMemsetAsync(scale, 0, n, st));
        const float floor_s = (fmt == FP8_E4M3 ? 1e-12f / 448.0f : 1e-12f / 57344.0f);
        return cuda_status(launch_fill_scale(static_cast<float*>(scale), n, floor_s, st));
    }
    return cuda_status(launch_quantize_grouped(a, st));
}

// An epilogue descriptor with every pointer NULL is the plain GEMM.
bool epi_active(const fp8_epilogue_t* e) {
    return e != nullptr && (e->bias_dev != nullptr || e->amax_dev != nullptr || e->yq_dev != nullptr);
}

int32_t check_epilogue(const fp8_epilogue_t* e, int64_t N) {
    if (!epi_active(e)) return FP8_OK;
    if (e->yq_dev != nullptr) {
        if (e->yq_fmt != FP8_E4M3 && e->yq_fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
        if (e->yq_scale_dev == nullptr || e->ldq < N) return FP8_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(e->yq_scale_dev) & 3u) != 0) return FP8_ERR_ALIGNMENT;
    }
    if (!aligned16(e->bias_dev)) return FP8_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(e->amax_dev) & 3u) != 0) return FP8_ERR_ALIGNMENT;
    return FP8_OK;
}

int32_t check_gemm_args(const uint8_t* a, const void* sa, int32_t am, int32_t fa, const uint8_t* b, const void* sb,
                        int32_t bm, int32_t fb, int64_t M, int64_t N, int64_t K, const void* y, int64_t ldy,
                        const fp8_epilogue_t* epi = nullptr) {
    if (fa != FP8_E4M3 && fa != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (fb != FP8_E4M3 && fb != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0) return FP8_ERR_INVALID_ARG;
    if (M >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31)) return FP8_ERR_INVALID_ARG;
    if (K % 16 != 0) return FP8_ERR_INVALID_ARG;
    auto pt_or_row = [](int32_t m) {
        return m == FP8_SCALE_TENSOR || m == FP8_SCALE_DELAYED || m == FP8_SCALE_ROW;
    };
    const bool rowscale = pt_or_row(am) && pt_or_row(bm);
    const bool block = am == FP8_SCALE_BLOCK_1x128 && bm == FP8_SCALE_BLOCK_128x128;
    const bool mx = am == FP8_SCALE_MX32 && bm == FP8_SCALE_MX32;
    if (!rowscale && !block && !mx) return FP8_ERR_INVALID_ARG;
    if (mx && (fa != FP8_E4M3 || fb != FP8_E4M3 || K % 32 != 0)) return FP8_ERR_INVALID_ARG;
    const bool fp8_only = y == nullptr && epi_active(epi) && epi->yq_dev != nullptr;
    if (!fp8_only && ldy < N) return FP8_ERR_INVALID_ARG;
    if (int32_t rc = check_epilogue(epi, N)) return rc;
    if (M > 0 && N > 0) {
        if (y == nullptr && !fp8_only) return FP8_ERR_INVALID_ARG;
        if (K > 0 && (a == nullptr || b == nullptr || sa == nullptr || sb == nullptr)) return FP8_ERR_INVALID_ARG;
    }
    if (!aligned16(a) || !aligned16(b) || (reinterpret_cast<uintptr_t>(y) & 1u) != 0) return FP8_ERR_ALIGNMENT;
    if (!mx && (((reinterpret_cast<uintptr_t>(sa) | reinterpret_cast<uintptr_t>(sb)) & 3u) != 0)) return FP8_ERR_ALIGNMENT;
    return FP8_OK;
}

int32_t gemm_impl(const uint8_t* a, const void* sa, int32_t am, int32_t fa, const uint8_t* b, const void* sb,
                  int32_t bm, int32_t fb, int64_t M, int64_t N, int64_t K, void* y, int64_t ldy, int32_t* status,
                  cudaStream_t st, const fp8_epilogue_t* epi = nullptr, bool a_just_quantized = false) {
    if (M == 0 || N == 0) return FP8_OK;
    const bool ext = epi_active(epi);
    if (K == 0 && !ext) return cuda_status(launch_zero_output(static_cast<uint16_t*>(y), M, N, ldy, st));
    GemmArgs g{};
    if (ext) {
        g.bias = static_cast<const uint16_t*>(epi->bias_dev);
        g.amax = epi->amax_dev;
        g.yq = epi->yq_dev;
        g.yq_scale = epi->yq_scale_dev;
        g.yq_fmt = epi->yq_fmt;
        g.ldq = epi->ldq;
    }
    g.a = a;
    g.b = b;
    g.sa = sa;
    g.sb = sb;
    g.a_mode = am;
    g.b_mode = bm;
    g.fmt_a = fa;
    g.fmt_b = fb;
    g.M = M;
    g.N = N;
    g.K = K;
    g.y = static_cast<uint16_t*>(y);
    g.ldy = ldy;
    g.status = status;
    g.a_from_previous_kernel = a_just_quantized;
    if (K == 0) return cuda_status(launch_zero_k_epilogue(g, st));
    return cuda_status(launch_gemm(g, st));
}

}  // namespace

extern "C" {

int32_t fp8_abi_version(void) { return FP8_ABI_VERSION; }

const char* fp8_status_string(int32_t s) {
    switch (s) {
    case FP8_OK: return "FP8_OK";
    case FP8_ERR_INVALID_ARG: return "FP8_ERR_INVALID_ARG";
    case FP8_ERR_ALIGNMENT: return "FP8_ERR_ALIGNMENT";
    case FP8_ERR_UNSUPPORTED_DEVICE: return "FP8_ERR_UNSUPPORTED_DEVICE";
    case FP8_ERR_NONFINITE: return "FP8_ERR_NONFINITE";
    case FP8_ERR_TIMEOUT: return "FP8_ERR_TIMEOUT";
    case FP8_ERR_CUDA: return "FP8_ERR_CUDA";
    case FP8_ERR_WORKSPACE: return "FP8_ERR_WORKSPACE";
    default: return "FP8_ERR_UNKNOWN";
    }
}

int32_t fp8_device_check(void) { return device_gate(); }

void fp8_testing_set_wait_limit_ns(uint64_t ns) { set_wait_limit_ns(ns); }

int32_t fp8_testing_encode_f32_range(uint32_t first_bits, int64_t n, int32_t fmt, uint8_t* q, void* stream) {
    if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (n < 0 || (uint64_t)first_bits + (uint64_t)n > ((uint64_t)1 << 32)) return FP8_ERR_INVALID_ARG;
    if (n == 0) return FP8_OK;
    if (q == nullptr) return FP8_ERR_INVALID_ARG;
    const int32_t gate = device_gate();
    if (gate != FP8_OK) return gate;
    return cuda_status(launch_encode_f32_range(first_bits, n, fmt, q, static_cast<cudaStream_t>(stream)));
}

size_t fp8_workspace_size(int32_t which, int64_t M, int64_t N, int64_t K, int32_t mode) {
    (void)N;
    if (which == 0) return (mode == FP8_SCALE_TENSOR || mode == FP8_SCALE_DELAYED) ? partials_bytes() : 0;
    if (which == 1) return 0;
    if (which == 2) {
        if (M < 0 || K < 0) return 0;
        const int64_t sb = scale_bytes(mode, M, K);
        if (sb < 0) return 0;
        return align_up((size_t)(M * K), 256) + align_up((size_t)sb, 256) + partials_bytes();
    }
    return 0;
}

int32_t fp8_quantize(const void* x_dev, int64_t rows, int64_t cols, int64_t ld, int32_t fmt, int32_t mode,
                     uint8_t* q_dev, void* scale_dev, fp8_history_t* hist, void* dequant_dev, int32_t* dev_status,
                     void* workspace_dev, size_t ws_bytes, void* stream) {
    int32_t rc = check_quantize_args(x_dev, rows, cols, ld, fmt, mode, q_dev, scale_dev, hist, dequant_dev);
    if (rc != FP8_OK) return rc;
    if ((rc = device_gate()) != FP8_OK) return rc;
    return quantize_impl(x_dev, rows, cols, ld, fmt, mode, q_dev, scale_dev, hist, dequant_dev, dev_status,
                         workspace_dev, ws_bytes, static_cast<cudaStream_t>(stream));
}

int32_t fp8_amax(const void* x_dev, int64_t rows, int64_t cols, int64_t ld, float* amax_dev, int32_t* dev_status,
                 void* workspace_dev, size_t ws_bytes, void* stream) {
    if (amax_dev == nullptr) return FP8_ERR_INVALID_ARG;
    int32_t rc = check_quantize_args(x_dev, rows, cols, ld, FP8_E4M3, FP8_SCALE_TENSOR, nullptr, amax_dev, nullptr,
                                     nullptr, /*need_q=*/false);
    if (rc != FP8_OK) return rc;
    if ((rc = device_gate()) != FP8_OK) return rc;
    if (workspace_dev == nullptr || ws_bytes < partials_bytes()) return FP8_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace_dev) & 3u) != 0) return FP8_ERR_ALIGNMENT;
    QuantArgs a{};
    a.x = static_cast<const uint16_t*>(x_dev);
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.status = dev_status;
    a.partials = static_cast<uint32_t*>(workspace_dev);
    return cuda_status(launch_amax(a, amax_dev, static_cast<cudaStream_t>(stream)));
}

int32_t fp8_quantize_with_amax(const void* x_dev, int64_t rows, int64_t cols, int64_t ld, int32_t fmt,
                               const float* amax_dev, uint8_t* q_dev, float* scale_dev, void* dequant_dev,
                               int32_t* dev_status, void* stream) {
    if (amax_dev == nullptr || scale_dev == nullptr) return FP8_ERR_INVALID_ARG;
    int32_t rc = check_quantize_args(x_dev, rows, cols, ld, fmt, FP8_SCALE_TENSOR, q_dev, scale_dev, nullptr,
                                     dequant_dev);
    if (rc != FP8_OK) return rc;
    if ((reinterpret_cast<uintptr_t>(amax_dev) & 3u) != 0) return FP8_ERR_ALIGNMENT;
    if ((rc = device_gate()) != FP8_OK) return rc;
    QuantArgs a{};
    a.x = static_cast<const uint16_t*>(x_dev);
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.fmt = fmt;
    a.mode = FP8_SCALE_TENSOR;
    a.q = q_dev;
    a.scale = scale_dev;
    a.deq = static_cast<uint16_t*>(dequant_dev);
    a.status = dev_status;
    a.amax_in = amax_dev;
    return cuda_status(launch_quantize_given(a, static_cast<cudaStream_t>(stream)));
}

int32_t fp8_scaled_gemm(const uint8_t* a_dev, const void* a_scale_dev, int32_t a_mode, int32_t fmt_a,
                        const uint8_t* b_dev, const void* b_scale_dev, int32_t b_mode, int32_t fmt_b, int64_t M,
                        int64_t N, int64_t K, void* y_dev, int64_t ldy, int32_t* dev_status, void* workspace_dev,
                        size_t ws_bytes, void* stream) {
    (void)workspace_dev;
    (void)ws_bytes;
    int32_t rc = check_gemm_args(a_dev, a_scale_dev, a_mode, fmt_a, b_dev, b_scale_dev, b_mode, fmt_b, M, N, K, y_dev,
                                 ldy);
    if (rc != FP8_OK) return rc;
    if ((rc = device_gate()) != FP8_OK) return rc;
    return gemm_impl(a_dev, a_scale_dev, a_mode, fmt_a, b_dev, b_scale_dev, b_mode, fmt_b, M, N, K, y_dev, ldy,
                     dev_status, static_cast<cudaStream_t>(stream));
}

int32_t fp8_scaled_gemm_ex(const uint8_t* a_dev, const void* a_scale_dev, int32_t a_mode, int32_t fmt_a,
                           const uint8_t* b_dev, const void* b_scale_dev, int32_t b_mode, int32_t fmt_b, int64_t M,
                           int64_t N, int64_t K, void* y_dev, int64_t ldy, const fp8_epilogue_t* epi,
                           int32_t* dev_status, void* workspace_dev, size_t ws_bytes, void* stream) {
    (void)workspace_dev;
    (void)ws_bytes;
    int32_t rc = check_gemm_args(a_dev, a_scale_dev, a_mode, fmt_a, b_dev, b_scale_dev, b_mode, fmt_b, M, N, K, y_dev,
                                 ldy, epi);
    if (rc != FP8_OK) return rc;
    if ((rc = device_gate()) != FP8_OK) return rc;
    return gemm_impl(a_dev, a_scale_dev, a_mode, fmt_a, b_dev, b_scale_dev, b_mode, fmt_b, M, N, K, y_dev, ldy,
                     dev_status, static_cast<cudaStream_t>(stream), epi);
}

int32_t fp8_weight_only_linear(const void* x_dev, int64_t M, int64_t K, int64_t ldx, const uint8_t* w_dev,
                               const void* w_scale_dev, int32_t w_mode, int32_t w_fmt, int64_t N, void* y_dev,
                               int64_t ldy, int32_t* dev_status, void* stream) {
    if (w_fmt != FP8_E4M3 && w_fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (w_mode != FP8_SCALE_TENSOR && w_mode != FP8_SCALE_ROW && w_mode != FP8_SCALE_DELAYED) return FP8_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0 || M > FP8_WEIGHT_ONLY_MAX_TOKENS) return FP8_ERR_INVALID_ARG;
    if (N >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31)) return FP8_ERR_INVALID_ARG;
    if (K % 16 != 0 || ldy < N || (K > 0 && ldx < K)) return FP8_ERR_INVALID_ARG;
    if (M > 0 && N > 0) {
        if (y_dev == nullptr) return FP8_ERR_INVALID_ARG;
        if (K > 0 && (x_dev == nullptr || w_dev == nullptr || w_scale_dev == nullptr)) return FP8_ERR_INVALID_ARG;
    }
    // X and W are not read when K == 0
    if (K > 0 && (ldx % 8 != 0 || !aligned16(x_dev) || !aligned16(w_dev))) return FP8_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(w_scale_dev) & 3u) != 0 || (reinterpret_cast<uintptr_t>(y_dev) & 1u) != 0)
        return FP8_ERR_ALIGNMENT;
    int32_t rc = device_gate();
    if (rc != FP8_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (M == 0 || N == 0) return FP8_OK;
    if (K == 0) return cuda_status(launch_zero_output(static_cast<uint16_t*>(y_dev), M, N, ldy, st));
    WoArgs g{};
    g.x = static_cast<const uint16_t*>(x_dev);
    g.ldx = ldx;
    g.w = w_dev;
    g.sw = w_scale_dev;
    g.w_row_scales = w_mode == FP8_SCALE_ROW;
    g.w_fmt = w_fmt;
    g.M = M;
    g.N = N;
    g.K = K;
    g.y = static_cast<uint16_t*>(y_dev);
    g.ldy = ldy;
    g.status = dev_status;
    return cuda_status(launch_weight_only(g, st));
}

int32_t fp8_linear_forward_ex(const void* x_dev, int64_t M, int64_t K, int64_t ldx, int32_t x_fmt, int32_t x_mode,
                           fp8_history_t* hist, const uint8_t* w_dev, const void* w_scale_dev, int32_t w_mode,
                              int32_t w_fmt, int64_t N, void* y_dev, int64_t ldy, const fp8_epilogue_t* epi,
                              int32_t* dev_status, void* workspace_dev, size_t ws_bytes, void* stream) {
    if (x_mode == FP8_SCALE_BLOCK_128x128) return FP8_ERR_INVALID_ARG;   // activations use 1x128 blocks
    const size_t need = fp8_workspace_size(2, M, N, K, x_mode);
    if (need == 0) return FP8_ERR_INVALID_ARG;
    if (workspace_dev == nullptr || ws_bytes < need) return FP8_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace_dev) & 255u) != 0) return FP8_ERR_ALIGNMENT;
    uint8_t* ws = static_cast<uint8_t*>(workspace_dev);
    uint8_t* xq = ws;
    void* xs = ws + align_up((size_t)(M * K), 256);
    void* part = ws + align_up((size_t)(M * K), 256) + align_up((size_t)scale_bytes(x_mode, M, K), 256);
    int32_t rc = check_quantize_args(x_dev, M, K, ldx, x_fmt, x_mode, xq, xs, hist, nullptr);
    if (rc != FP8_OK) return rc;
    const int32_t gm_a = x_mode == FP8_SCALE_DELAYED ? FP8_SCALE_TENSOR : x_mode;
    rc = check_gemm_args(xq, xs, gm_a, x_fmt, w_dev, w_scale_dev, w_mode, w_fmt, M, N, K, y_dev, ldy, epi);
    if (rc != FP8_OK) return rc;
    if ((rc = device_gate()) != FP8_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = quantize_impl(x_dev, M, K, ldx, x_fmt, x_mode, xq, xs, hist, nullptr, dev_status, part, partials_bytes(), st);
    if (rc != FP8_OK) return rc;
    // the quantize kernel just enqueued wrote X's codes and scales and nothing else
    return gemm_impl(xq, xs, gm_a, x_fmt, w_dev, w_scale_dev, w_mode, w_fmt, M, N, K, y_dev, ldy, dev_status, st, epi,
                     /*a_just_quantized=*/true);
}

int32_t fp8_linear_forward(const void* x_dev, int64_t M, int64_t K, int64_t ldx, int32_t x_fmt, int32_t x_mode,
                           fp8_history_t* hist, const uint8_t* w_dev, const void* w_scale_dev, int32_t w_mode,
                           int32_t w_fmt, int64_t N, void* y_dev, int64_t ldy, int32_t* dev_status,
                           void* workspace_dev, size_t ws_bytes, void* stream) {
    return fp8_linear_forward_ex(x_dev, M, K, ldx, x_fmt, x_mode, hist, w_dev, w_scale_dev, w_mode, w_fmt, N, y_dev,
                                 ldy, nullptr, dev_status, workspace_dev, ws_bytes, stream);
}

}  // extern "C"
