// noalloc.cu -- fp8_linear_forward_noalloc: the FP8 linear forward for callers
// that cannot allocate device memory.
//
// Who needs this: code that runs inside a host program which owns every device
// allocation and hands its plug-ins only their input and output buffers (no
// allocator, no workspace), and callers for which a cudaMalloc -- which may
// synchronise the whole device -- is not acceptable on their path.  For them the
// scratch that fp8_linear_forward takes as `workspace` (the quantised activations,
// their scales and the per-tensor amax partials) lives in one fixed array of
// device memory that is part of this library.
//
// The array: FP8_NOALLOC_SCRATCH_BYTES (4 MiB) per GPU, reserved on every GPU on
// which the library's device code is loaded and kept until the process exits.
// Nothing in it has to start at zero: every call writes each scratch byte it later
// reads.  All calls share it and it keeps the last call's contents, so two calls
// whose work overlaps on the GPU (different streams, or different host threads
// without ordering) race on it and may corrupt each other's results.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

// File-scope scratch for the no-allocation entry point.  Host code must not use
// the name as an address: it only stands for the device symbol, whose device
// address is fetched with cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_linear_scratch[FP8_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices];   // device address of g_linear_scratch, per device

// Once per device, with that device current: look up the scratch's device address.
int32_t scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP8_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FP8_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_linear_scratch) != cudaSuccess || p == nullptr) return FP8_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return FP8_OK;
}

}  // namespace

extern "C" {

int32_t fp8_linear_forward_noalloc(const void* x_dev, int64_t M, int64_t K, int64_t ldx, int32_t x_fmt,
                                   int32_t x_mode, fp8_history_t* hist, const uint8_t* w_dev,
                                   const void* w_scale_dev, int32_t w_mode, int32_t w_fmt, int64_t N, void* y_dev,
                                   int64_t ldy, int32_t* dev_status, void* stream) {
    const size_t need = fp8_workspace_size(2, M, N, K, x_mode);
    if (need == 0) return FP8_ERR_INVALID_ARG;
    if (need > (size_t)FP8_NOALLOC_SCRATCH_BYTES) return FP8_ERR_WORKSPACE;   // input too large for the fixed scratch
    int32_t rc = fp8_device_check();
    if (rc != FP8_OK) return rc;
    void* scratch = nullptr;
    if ((rc = scratch_for_current_device(&scratch)) != FP8_OK) return rc;
    return fp8_linear_forward(x_dev, M, K, ldx, x_fmt, x_mode, hist, w_dev, w_scale_dev, w_mode, w_fmt, N, y_dev,
                              ldy, dev_status, scratch, (size_t)FP8_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
