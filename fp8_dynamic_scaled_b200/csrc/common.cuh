// common.cuh -- device helpers shared by the quantize and GEMM kernels of libfp8.
// sm_100a only.  Built without fast-math: fp32 division is IEEE, no FTZ.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fp8.h"

namespace fp8b {

// Largest finite magnitude of each format ([FFS] section "8 个 Bit 怎样分配").
template <int FMT>
__host__ __device__ constexpr float fmax_of() {
    return FMT == FP8_E4M3 ? 448.0f : 57344.0f;
}

// Floor on amax before the scale division ([PQG] code: clamp(amax, min=1e-12)).
__host__ __device__ constexpr float amax_floor() { return 1e-12f; }

// s = fp32(max(amax, 1e-12f) / F_max), an IEEE division.
template <int FMT>
__device__ __forceinline__ float scale_from_amax(float amax) {
    return __fdiv_rn(fmaxf(amax, amax_floor()), fmax_of<FMT>());
}

// ---------------------------------------------------------------- bf16 helpers
// |x| of the two bf16 values packed in a 32-bit word, as 16-bit patterns.  For
// non-negative bf16 patterns, unsigned integer order equals value order, and
// every NaN/Inf pattern (>= 0x7F80) is above every finite one.
__device__ __forceinline__ uint32_t abs_bf16x2(uint32_t w) { return w & 0x7FFF7FFFu; }

__device__ __forceinline__ uint32_t max_bf16x2_bits(uint32_t a, uint32_t b) { return __vmaxu2(a, b); }

// Reduce a packed pair of |bf16| patterns to one 16-bit pattern.
__device__ __forceinline__ uint32_t hmax_pair(uint32_t w) {
    uint32_t lo = w & 0xFFFFu, hi = w >> 16;
    return lo > hi ? lo : hi;
}

__device__ __forceinline__ float bf16bits_to_float(uint32_t b16) { return __uint_as_float(b16 << 16); }

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Lane-wise max of |a|, |b| on packed bf16 pairs; NaN in either input gives NaN
// (the sign bits of the result are the xor of the inputs' signs: mask them off).
__device__ __forceinline__ uint32_t bmax_abs_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Packed fp32 pair arithmetic (one instruction for two lanes), round to nearest.
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
    float2 d;
    asm("mul.rn.f32x2 %0, %1, %2;"
        : "=l"(reinterpret_cast<unsigned long long&>(d))
        : "l"(reinterpret_cast<const unsigned long long&>(a)), "l"(reinterpret_cast<const unsigned long long&>(b)));
    return d;
}
__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
    float2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(reinterpret_cast<unsigned long long&>(d))
        : "l"(reinterpret_cast<const unsigned long long&>(a)), "l"(reinterpret_cast<const unsigned long long&>(b)),
          "l"(reinterpret_cast<const unsigned long long&>(c)));
    return d;
}

__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
    float2 d;
    asm("add.rn.f32x2 %0, %1, %2;"
        : "=l"(reinterpret_cast<unsigned long long&>(d))
        : "l"(reinterpret_cast<const unsigned long long&>(a)), "l"(reinterpret_cast<const unsigned long long&>(b)));
    return d;
}

// Lane-wise clamp of a packed bf16 pair to [lo, hi] (both packed pairs).
__device__ __forceinline__ uint32_t clamp_bf16x2(uint32_t v, uint32_t lo, uint32_t hi) {
    uint32_t d;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(v), "r"(hi));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(d), "r"(lo));
    return d;
}

// ---------------------------------------------------------------- FP8 casts
// Two fp32 values -> two codes (a in the low byte), round-to-nearest-even with
// saturation to the largest finite value: for finite inputs identical to
// clip(+-F_max) followed by the RNE cast.
template <int FMT>
__device__ __forceinline__ uint32_t cvt_pair(float a, float b) {
    __nv_fp8x2_storage_t r = __nv_cvt_float2_to_fp8x2(
        make_float2(a, b), __NV_SATFINITE, FMT == FP8_E4M3 ? __NV_E4M3 : __NV_E5M2);
    return (uint32_t)r;
}

// Two codes (low byte first) -> two exact fp32 values.
template <int FMT>
__device__ __forceinline__ float2 decode_pair(uint32_t codes2) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(codes2 & 0xFFFFu),
                                              FMT == FP8_E4M3 ? __NV_E4M3 : __NV_E5M2);
    return __half22float2(*reinterpret_cast<__half2*>(&h));
}

// Two fp32 -> packed bf16x2 (RNE), a in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------- memory
__device__ __forceinline__ uint4 ld_v4(const void* p) {
    return *reinterpret_cast<const uint4*>(p);
}
__device__ __forceinline__ uint4 ld_v4_stream(const void* p) {
    return __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void st_v4_stream(void* p, uint4 v) {
    __stcs(reinterpret_cast<uint4*>(p), v);
}

// Programmatic dependent launch: let the next kernel in the stream (if it was
// launched as a programmatic dependent) start now; it waits for this grid's results
// with pdl_wait() before it reads them.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Wait until the preceding grid (if this one was launched as its programmatic
// dependent) has completed and its writes are visible; a no-op otherwise.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Host: the current device as an index into small per-device caches (kernel
// attributes, SM counts), or -1 when it is outside them (then nothing is cached).
constexpr int kDeviceCacheSlots = 64;
inline int device_slot() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kDeviceCacheSlots) return -1;
    return d;
}

// Record the first device-side error in a caller-owned status word.
__device__ __forceinline__ void report_status(int32_t* status, int32_t code) {
    if (status) atomicCAS(status, 0, code);
}

}  // namespace fp8b
