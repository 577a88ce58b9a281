// quantize.cu -- fused amax-reduce + scale + saturating RNE cast kernels (sm_100a).
//
// What is computed ([FFS] = "FP8 formats, scaling and LLM inference",
// [PQG] = "FP8 产线量化落地指南"):
//   a_max = max|x| over the scaling group          ([FFS] "Scale 怎样把 Tensor 塞进 E4M3", eq. a_max)
//   s     = fp32(max(a_max, 1e-12f) / F_max)      ([FFS] eq. s = a_max/F_max; [PQG] code)
//   q     = RNE_fp8(clip(fp32(x / s), +-F_max))   ([FFS] eq. X_fp8; [PQG] code step 3)
//   d     = bf16_RNE(fp32(decode(q) * s))         ([FFS] eq. X^ = s X_fp8), optional
// Groups: the whole tensor (TENSOR, DELAYED), a row (ROW), 1x128 and 128x128
// blocks ([FFS] "Per-channel 与 Block Scaling", eq. s_g = a_g/F_max), and 32-element
// MX blocks with a power-of-two scale 2^e, e = clamp(floor(log2 a_max) - 8, -127, 127).
//
// Data movement: every kernel reads bf16 with 16-byte vector loads that are
// contiguous across a warp, and writes codes with 8-byte stores that are
// contiguous across a warp.  amax is an integer max over the |bf16| bit
// patterns (exact and order-free); a pattern >= 0x7F80 flags NaN/Inf input.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace fp8b {

constexpr int QT = 256;     // threads per CTA of the streaming kernels
constexpr int VEC = 8;      // bf16 elements per 16-byte vector

// ---------------------------------------------------------------- per-vector ops
// |x| max over the 8 bf16 of a vector, as a packed pair of 16-bit patterns.
__device__ __forceinline__ uint32_t vec_amax2(const uint4& v) {
    uint32_t a = max_bf16x2_bits(abs_bf16x2(v.x), abs_bf16x2(v.y));
    uint32_t b = max_bf16x2_bits(abs_bf16x2(v.z), abs_bf16x2(v.w));
    return max_bf16x2_bits(a, b);
}

// How one element turns into the value that is cast: x / s (IEEE division) for
// fp32 scales, x * 2^-e (exact) for MX scales.
struct DivScale {
    float s;
    __device__ __forceinline__ float operator()(float x) const { return __fdiv_rn(x, s); }
    __device__ __forceinline__ float deq() const { return s; }
};
struct Pow2Scale {
    float inv;   // 2^-e
    float mul;   // 2^e
    __device__ __forceinline__ float operator()(float x) const { return __fmul_rn(x, inv); }
    __device__ __forceinline__ float deq() const { return mul; }
};

// 8 elements -> 8 codes (byte i = element i).
template <int FMT, class Op>
__device__ __forceinline__ uint2 cast_vec(const uint4& v, const Op& op) {
    uint32_t c0 = cvt_pair<FMT>(op(bf16_lo(v.x)), op(bf16_hi(v.x)));
    uint32_t c1 = cvt_pair<FMT>(op(bf16_lo(v.y)), op(bf16_hi(v.y)));
    uint32_t c2 = cvt_pair<FMT>(op(bf16_lo(v.z)), op(bf16_hi(v.z)));
    uint32_t c3 = cvt_pair<FMT>(op(bf16_lo(v.w)), op(bf16_hi(v.w)));
    return make_uint2(c0 | (c1 << 16), c2 | (c3 << 16));
}

// 8 codes -> 8 bf16 of decode(q) * mul.
template <int FMT>
__device__ __forceinline__ uint4 dequant_vec(const uint2& c, float mul) {
    float2 a = decode_pair<FMT>(c.x & 0xFFFFu);
    float2 b = decode_pair<FMT>(c.x >> 16);
    float2 d = decode_pair<FMT>(c.y & 0xFFFFu);
    float2 e = decode_pair<FMT>(c.y >> 16);
    return make_uint4(pack_bf16x2(__fmul_rn(a.x, mul), __fmul_rn(a.y, mul)),
                      pack_bf16x2(__fmul_rn(b.x, mul), __fmul_rn(b.y, mul)),
                      pack_bf16x2(__fmul_rn(d.x, mul), __fmul_rn(d.y, mul)),
                      pack_bf16x2(__fmul_rn(e.x, mul), __fmul_rn(e.y, mul)));
}

// MX shared exponent from an amax bf16 pattern: floor(log2 a) is the unbiased
// exponent of a (bf16 subnormals: position of the leading mantissa bit).
__device__ __forceinline__ int mx_exponent(uint32_t amax_bits) {
    if (amax_bits == 0) return -127;
    int ebits = (int)(amax_bits >> 7) & 0xFF;
    int flog2;
    if (ebits != 0) {
        flog2 = ebits - 127;
    } else {
        int m = (int)(amax_bits & 0x7F);               // subnormal: m * 2^-133
        flog2 = (31 - __clz(m)) - 133;
    }
    int e = flog2 - 8;
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^k as an fp32 value for k in [-149, 127] (exact).
__device__ __forceinline__ float exp2i(int k) {
    if (k >= -126) return __uint_as_float((uint32_t)(k + 127) << 23);
    return __uint_as_float(1u << (k + 149));
}

// Block-wide max of a 32-bit pattern (all threads get the result).
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t* red /* [32] */) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    const int nw = blockDim.x >> 5;
    uint32_t r = lane < nw ? red[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) r = max(r, __shfl_xor_sync(0xffffffffu, r, o));
    return r;
}

// A caller-supplied amax (fp8_quantize_with_amax): NaN or +Inf is reported and
// replaced by the largest finite fp32 so that the scale stays finite.
__device__ __forceinline__ float given_amax(const float* a, int32_t* status) {
    float v = *a;
    if (!(v <= 3.402823466e38f)) {
        if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) report_status(status, FP8_ERR_NONFINITE);
        v = 3.402823466e38f;
    }
    return v;
}

// ================================================================ per-tensor
// Phase 1: each CTA writes the max |bf16| pattern over its share of the tensor.
// The tensor is viewed as nrows rows of nvec 16-byte vectors (a dense tensor is
// passed as one long row).
__global__ void __launch_bounds__(QT) amax_partials_kernel(const uint16_t* __restrict__ x, int64_t nrows,
                                                           int64_t nvec, int64_t ld,
                                                           uint32_t* __restrict__ partials) {
    pdl_launch_dependents();   // a dependent GEMM may start streaming its other operand
    __shared__ uint32_t red[32];
    uint32_t m2 = 0;
    const int64_t stride = (int64_t)gridDim.x * QT;
    for (int64_t r = blockIdx.y; r < nrows; r += gridDim.y) {
        const uint16_t* row = x + r * ld;
        int64_t v = (int64_t)blockIdx.x * QT + threadIdx.x;
        for (; v + 3 * stride < nvec; v += 4 * stride) {
            uint4 a = ld_v4(row + v * VEC);
            uint4 b = ld_v4(row + (v + stride) * VEC);
            uint4 c = ld_v4(row + (v + 2 * stride) * VEC);
            uint4 d = ld_v4(row + (v + 3 * stride) * VEC);
            m2 = max_bf16x2_bits(m2, max_bf16x2_bits(max_bf16x2_bits(vec_amax2(a), vec_amax2(b)),
                                                     max_bf16x2_bits(vec_amax2(c), vec_amax2(d))));
        }
        for (; v < nvec; v += stride) m2 = max_bf16x2_bits(m2, vec_amax2(ld_v4(row + v * VEC)));
    }
    uint32_t m = block_max_u32(hmax_pair(m2), red);
    if (threadIdx.x == 0) partials[(int64_t)blockIdx.y * gridDim.x + blockIdx.x] = m;
}

// Phase 2 (current scaling) or the single pass (delayed scaling, t >= 1).
//   SRC_PARTIALS: s from the phase-1 partials (every CTA reduces them itself, so
//                 no counter or grid barrier is needed).  When ring != nullptr
//                 (delayed step 0) CTA 0 also records ring[slot] = amax.
//   SRC_RING:     s from max(ring); the CTAs also reduce amax_t of this input
//                 into *pending and the last CTA to finish (ticket) commits it to
//                 ring[slot] and rearms pending/ticket.
//   SRC_GIVEN:    s from a caller's amax (ring[0]); the cast checks for non-finite input.
enum { SRC_PARTIALS = 0, SRC_RING = 1, SRC_GIVEN = 2 };

template <int FMT, bool DEQ, int SRC>
__global__ void __launch_bounds__(QT) cast_tensor_kernel(
    const uint16_t* __restrict__ x, int64_t nrows, int64_t nvec, int64_t ld,
    const uint32_t* __restrict__ partials, int32_t npartials,
    float* ring, int32_t ring_len, int32_t slot, float* pending, uint32_t* ticket,
    uint8_t* __restrict__ q, float* __restrict__ scale_out, uint16_t* __restrict__ deq,
    int32_t* status) {
    pdl_launch_dependents();   // a dependent GEMM may start streaming its other operand
    __shared__ uint32_t red[32];
    // ---- the scale
    uint32_t src = 0;
    if (SRC == SRC_PARTIALS) {
        for (int i = threadIdx.x; i < npartials; i += QT) src = max(src, partials[i]);
    } else if (SRC == SRC_RING) {
        for (int i = threadIdx.x; i < ring_len; i += QT) src = max(src, __float_as_uint(ring[i]));
    }
    if (SRC != SRC_GIVEN) src = block_max_u32(src, red);
    float amax;
    bool finite_in = true;     // step 0 of a delayed history records only a finite amax
    if (SRC == SRC_PARTIALS) {
        if (src >= 0x7F80u) {
            if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) report_status(status, FP8_ERR_NONFINITE);
            src = 0x7F7Fu;     // keep the scale finite; outputs are unspecified then
            finite_in = false;
        }
        amax = bf16bits_to_float(src);
    } else if (SRC == SRC_RING) {
        amax = __uint_as_float(src);
    } else {
        amax = given_amax(ring, status);
    }
    const DivScale op{scale_from_amax<FMT>(amax)};
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
        scale_out[0] = op.s;
        if (SRC == SRC_PARTIALS && ring != nullptr && finite_in) ring[slot] = amax;
    }
    constexpr bool CHECK = SRC != SRC_PARTIALS;   // inputs not already scanned by phase 1
    // ---- the cast
    uint32_t m2 = 0;
    const int64_t stride = (int64_t)gridDim.x * QT;
    for (int64_t r = blockIdx.y; r < nrows; r += gridDim.y) {
        const uint16_t* row = x + r * ld;
        uint8_t* qrow = q + r * (nvec * VEC);
        uint16_t* drow = DEQ ? deq + r * (nvec * VEC) : nullptr;
        int64_t v = (int64_t)blockIdx.x * QT + threadIdx.x;
        for (; v + stride < nvec; v += 2 * stride) {
            uint4 a = ld_v4(row + v * VEC);
            uint4 b = ld_v4(row + (v + stride) * VEC);
            if (CHECK) m2 = max_bf16x2_bits(m2, max_bf16x2_bits(vec_amax2(a), vec_amax2(b)));
            uint2 ca = cast_vec<FMT>(a, op), cb = cast_vec<FMT>(b, op);
            *reinterpret_cast<uint2*>(qrow + v * VEC) = ca;
            *reinterpret_cast<uint2*>(qrow + (v + stride) * VEC) = cb;
            if (DEQ) {
                st_v4_stream(drow + v * VEC, dequant_vec<FMT>(ca, op.s));
                st_v4_stream(drow + (v + stride) * VEC, dequant_vec<FMT>(cb, op.s));
            }
        }
        for (; v < nvec; v += stride) {
            uint4 a = ld_v4(row + v * VEC);
            if (CHECK) m2 = max_bf16x2_bits(m2, vec_amax2(a));
            uint2 ca = cast_vec<FMT>(a, op);
            *reinterpret_cast<uint2*>(qrow + v * VEC) = ca;
            if (DEQ) st_v4_stream(drow + v * VEC, dequant_vec<FMT>(ca, op.s));
        }
    }
    if (SRC == SRC_GIVEN) {
        const uint32_t m = block_max_u32(hmax_pair(m2), red);
        if (threadIdx.x == 0 && m >= 0x7F80u) report_status(status, FP8_ERR_NONFINITE);
    }
    if (SRC == SRC_RING) {
        uint32_t m = block_max_u32(hmax_pair(m2), red);
        if (threadIdx.x == 0) {
            if (m >= 0x7F80u) report_status(status, FP8_ERR_NONFINITE);
            // amax >= 0, so the fp32 bit pattern orders like the value
            atomicMax(reinterpret_cast<uint32_t*>(pending), m << 16);
            __threadfence();
            const uint32_t total = gridDim.x * gridDim.y;
            uint32_t t = atomicAdd(ticket, 1u);
            if (t == total - 1) {
                // every CTA has read the ring (they all did so before taking a ticket);
                // a step that saw a NaN/Inf records nothing: its slot keeps the old amax
                __threadfence();
                uint32_t a_t = atomicOr(reinterpret_cast<uint32_t*>(pending), 0u);
                if (a_t < 0x7F800000u) ring[slot] = __uint_as_float(a_t);
                *reinterpret_cast<volatile uint32_t*>(pending) = 0u;
                *reinterpret_cast<volatile uint32_t*>(ticket) = 0u;
            }
        }
    }
}

// ================================================================ segment kernels
// ROW (short rows), BLOCK_1x128 and MX32: a group of G lanes (inside one warp)
// owns one segment (a run of seg_vec vectors of one row) at a time; each lane
// holds up to U vectors of it in registers, so x is read exactly once.
//   FLAT: dense tensor whose rows split into whole segments; segment s starts at
//         element s*seg_vec*8 and owns scale s.
template <int FMT, bool DEQ, int G, int U, bool MX, bool FLAT>
__global__ void __launch_bounds__(QT) quant_segment_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    int32_t seg_vec, int64_t nseg_per_row, int64_t nseg,
    uint8_t* __restrict__ q, void* __restrict__ scale, uint16_t* __restrict__ deq, int32_t* status) {
    pdl_launch_dependents();   // a dependent GEMM may start streaming its other operand
    const int lane_g = threadIdx.x & (G - 1);
    const int64_t group = ((int64_t)blockIdx.x * QT + threadIdx.x) / G;
    const int64_t ngroups = (int64_t)gridDim.x * (QT / G);
    const unsigned gmask = G == 32 ? 0xffffffffu : (((1u << G) - 1u) << ((threadIdx.x & 31) & ~(G - 1)));
    for (int64_t s = group; s < nseg; s += ngroups) {
        int64_t row, c0;
        int32_t len_vec;
        if (FLAT) {
            row = 0; c0 = s * (int64_t)seg_vec * VEC; len_vec = seg_vec;
        } else {
            row = s / nseg_per_row;
            c0 = (s - row * nseg_per_row) * (int64_t)seg_vec * VEC;
            int64_t rem = (cols - c0) / VEC;
            len_vec = rem < seg_vec ? (int32_t)rem : seg_vec;
        }
        const uint16_t* src = x + row * ld + c0;
        uint4 v[U];
        uint32_t m2 = 0;
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int k = lane_g + G * i;
            if (k < len_vec) {
                v[i] = ld_v4_stream(src + (int64_t)k * VEC);
                m2 = max_bf16x2_bits(m2, vec_amax2(v[i]));
            }
        }
        uint32_t m = hmax_pair(m2);
#pragma unroll
        for (int o = G / 2; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(gmask, m, o));
        if (m >= 0x7F80u) {
            if (lane_g == 0) report_status(status, FP8_ERR_NONFINITE);
            m = 0x7F7Fu;
        }
        uint8_t* dst = q + row * cols + c0;
        uint16_t* ddst = DEQ ? deq + row * cols + c0 : nullptr;
        if (MX) {
            const int e = mx_exponent(m);
            const Pow2Scale op{exp2i(-e), exp2i(e)};
            if (lane_g == 0) reinterpret_cast<uint8_t*>(scale)[s] = (uint8_t)(e + 127);
#pragma unroll
            for (int i = 0; i < U; ++i) {
                const int k = lane_g + G * i;
                if (k < len_vec) {
                    uint2 c = cast_vec<FMT>(v[i], op);
                    *reinterpret_cast<uint2*>(dst + (int64_t)k * VEC) = c;
                    if (DEQ) st_v4_stream(ddst + (int64_t)k * VEC, dequant_vec<FMT>(c, op.deq()));
                }
            }
        } else {
            const DivScale op{scale_from_amax<FMT>(bf16bits_to_float(m))};
            if (lane_g == 0) reinterpret_cast<float*>(scale)[s] = op.s;
#pragma unroll
            for (int i = 0; i < U; ++i) {
                const int k = lane_g + G * i;
                if (k < len_vec) {
                    uint2 c = cast_vec<FMT>(v[i], op);
                    *reinterpret_cast<uint2*>(dst + (int64_t)k * VEC) = c;
                    if (DEQ) st_v4_stream(ddst + (int64_t)k * VEC, dequant_vec<FMT>(c, op.s));
                }
            }
        }
    }
}

// ROW with long rows: one CTA per row.  Rows of up to QT*UR vectors stay in
// registers (single pass); longer rows take a second pass for the cast.
template <int FMT, bool DEQ, int UR>
__global__ void __launch_bounds__(QT) quant_row_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                       int64_t cols, int64_t ld, uint8_t* __restrict__ q,
                                                       float* __restrict__ scale, uint16_t* __restrict__ deq,
                                                       int32_t* status) {
    pdl_launch_dependents();   // a dependent GEMM may start streaming its other operand
    __shared__ uint32_t red[32];
    const int64_t nvec = cols / VEC;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const uint16_t* src = x + r * ld;
        uint4 v[UR];
        uint32_t m2 = 0;
#pragma unroll
        for (int i = 0; i < UR; ++i) {
            const int64_t k = threadIdx.x + (int64_t)QT * i;
            if (k < nvec) {
                v[i] = ld_v4_stream(src + k * VEC);
                m2 = max_bf16x2_bits(m2, vec_amax2(v[i]));
            }
        }
        for (int64_t k = threadIdx.x + (int64_t)QT * UR; k < nvec; k += QT)
            m2 = max_bf16x2_bits(m2, vec_amax2(ld_v4(src + k * VEC)));
        uint32_t m = block_max_u32(hmax_pair(m2), red);
        if (m >= 0x7F80u) {
            if (threadIdx.x == 0) report_status(status, FP8_ERR_NONFINITE);
            m = 0x7F7Fu;
        }
        const DivScale op{scale_from_amax<FMT>(bf16bits_to_float(m))};
        if (threadIdx.x == 0) scale[r] = op.s;
        uint8_t* dst = q + r * cols;
        uint16_t* ddst = DEQ ? deq + r * cols : nullptr;
#pragma unroll
        for (int i = 0; i < UR; ++i) {
            const int64_t k = threadIdx.x + (int64_t)QT * i;
            if (k < nvec) {
                uint2 c = cast_vec<FMT>(v[i], op);
                *reinterpret_cast<uint2*>(dst + k * VEC) = c;
                if (DEQ) st_v4_stream(ddst + k * VEC, dequant_vec<FMT>(c, op.s));
            }
        }
        for (int64_t k = threadIdx.x + (int64_t)QT * UR; k < nvec; k += QT) {
            uint2 c = cast_vec<FMT>(ld_v4(src + k * VEC), op);
            *reinterpret_cast<uint2*>(dst + k * VEC) = c;
            if (DEQ) st_v4_stream(ddst + k * VEC, dequant_vec<FMT>(c, op.s));
        }
        __syncthreads();   // red[] is reused by the next row
    }
}

// BLOCK_128x128: one CTA per 128 x 128 tile; the 2048 vectors of a full tile sit
// in registers (8 per thread), rows of the tile are read by 16 consecutive lanes.
template <int FMT, bool DEQ>
__global__ void __launch_bounds__(QT) quant_block128_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                            int64_t cols, int64_t ld, uint8_t* __restrict__ q,
                                                            float* __restrict__ scale, uint16_t* __restrict__ deq,
                                                            int32_t* status) {
    pdl_launch_dependents();   // a dependent GEMM may start streaming its other operand
    __shared__ uint32_t red[32];
    constexpr int UB = 128 * 16 / QT;   // 8 vectors per thread
    const int64_t ncb = (cols + 127) / 128;
    const int64_t r0 = (int64_t)blockIdx.y * 128, c0 = (int64_t)blockIdx.x * 128;
    uint4 v[UB];
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < UB; ++i) {
        const int idx = threadIdx.x + QT * i;
        const int64_t r = r0 + (idx >> 4), c = c0 + (idx & 15) * VEC;
        if (r < rows && c < cols) {
            v[i] = ld_v4_stream(x + r * ld + c);
            m2 = max_bf16x2_bits(m2, vec_amax2(v[i]));
        }
    }
    uint32_t m = block_max_u32(hmax_pair(m2), red);
    if (m >= 0x7F80u) {
        if (threadIdx.x == 0) report_status(status, FP8_ERR_NONFINITE);
        m = 0x7F7Fu;
    }
    const DivScale op{scale_from_amax<FMT>(bf16bits_to_float(m))};
    if (threadIdx.x == 0) scale[(int64_t)blockIdx.y * ncb + blockIdx.x] = op.s;
#pragma unroll
    for (int i = 0; i < UB; ++i) {
        const int idx = threadIdx.x + QT * i;
        const int64_t r = r0 + (idx >> 4), c = c0 + (idx & 15) * VEC;
        if (r < rows && c < cols) {
            uint2 cq = cast_vec<FMT>(v[i], op);
            *reinterpret_cast<uint2*>(q + r * cols + c) = cq;
            if (DEQ) st_v4_stream(deq + r * cols + c, dequant_vec<FMT>(cq, op.s));
        }
    }
}

// ================================================================ register-resident kernels
// The fast path for dense shapes.  Each thread loads all of its 16-byte vectors
// before using any (VPT or U independent loads in flight), the data stays in
// registers from the amax through the cast, and small register footprints keep
// 8 CTAs (2,048 threads) resident per SM, so every SM has >= 128 KB of loads in
// flight -- enough to cover HBM latency at full bandwidth.  (A design that staged
// chunks through a shared-memory ring with bulk asynchronous copies was measured
// slower on B200 for these kernels: 4.9 vs 6.1 TB/s per-token, 4.2 vs 6.1 TB/s for
// 1x128 blocks.)
//   RQ_ROW      one CTA per row (per-token / per-channel scale), VPT vectors per thread
//   RQ_B128     1x128 blocks: 16 consecutive lanes reduce one block
//   RQ_MX       MX32 blocks: 4 consecutive lanes reduce one block
//   RQ_AMAX     per-tensor phase 1: grid-stride max of |x|, one partial per CTA
//   RQ_CAST     per-tensor phase 2: s from the partials, cast in the reverse of
//               phase 1's order (its last reads are the likeliest L2 hits)
//   RQ_DELAYED  delayed scaling t >= 1: s from the ring, amax_t reduced on the fly
//               and committed to the ring by the last CTA to finish
// The division x / s is a reciprocal plus one Markstein correction step: with
// r = RN(1/s), q = RN(x r), e = RN(x - q s) (exact through the FMA),
// RN(q + e r) equals RN(x / s) for every quotient in the fp32 normal range (P.
// Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990).  Quotients below the normal range
// (|t| < 2^-126) may differ in their last bits, but every such t encodes to a
// signed zero in both FP8 formats.
//   RQ_GIVEN    per-tensor cast with a caller's amax (fp8_quantize_with_amax)
enum { RQ_ROW = 0, RQ_B128 = 1, RQ_MX = 2, RQ_AMAX = 3, RQ_CAST = 4, RQ_DELAYED = 5, RQ_GIVEN = 6 };

struct RcpScale {
    float s, r;
};
template <int FMT>
__device__ __forceinline__ RcpScale rcp_scale_from_amax_bits(uint32_t m) {
    const float s = scale_from_amax<FMT>(bf16bits_to_float(m));
    return RcpScale{s, __frcp_rn(s)};
}

// |x| max over the 8 bf16 of a vector with packed bf16 max (the sign bits of the
// result are meaningless; NaN propagates).
__device__ __forceinline__ uint32_t vec_amax2_bf(const uint4& v) {
    return bmax_abs_bf16x2(bmax_abs_bf16x2(v.x, v.y), bmax_abs_bf16x2(v.z, v.w));
}

// 8 elements -> 8 codes with the Markstein-corrected division on packed pairs.
// The arithmetic runs on -x with -r: q = RN((-x)(-r)) = RN(x r),
// e' = RN(q s + (-x)) = -RN(x - q s), t = RN(e' (-r) + q) = RN(q + (x - q s) r);
// working on -x also makes x = -0 come out as -0 (code 0x80).
template <int FMT>
__device__ __forceinline__ uint2 cast_vec_rcp(const uint4& v, const RcpScale& op) {
    const float2 s2 = make_float2(op.s, op.s);
    const float2 nr2 = make_float2(-op.r, -op.r);
    uint32_t c[4];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t wn = w[i] ^ 0x80008000u;
        const float2 nx = make_float2(__uint_as_float(wn << 16), __uint_as_float(wn & 0xFFFF0000u));
        const float2 q = mul2_rn(nx, nr2);
        const float2 e = fma2_rn(q, s2, nx);
        const float2 t = fma2_rn(e, nr2, q);
        c[i] = cvt_pair<FMT>(t.x, t.y);
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// The same for quotients that may leave the fp32 range (delayed scaling: the
// history scale can be far below the current amax).  An infinite first quotient
// saturates to +-F_max as it is and is not corrected (which would give NaN).
template <int FMT>
__device__ __forceinline__ uint2 cast_vec_rcp_guarded(const uint4& v, const RcpScale& op) {
    uint32_t c[4];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float t[2];
        const float xs[2] = {bf16_lo(w[i]), bf16_hi(w[i])};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float nx = -xs[h];
            const float q = __fmul_rn(nx, -op.r);
            const float e = __fmaf_rn(q, op.s, nx);
            t[h] = fabsf(q) <= 3.402823466e38f ? __fmaf_rn(e, -op.r, q) : q;
        }
        c[i] = cvt_pair<FMT>(t[0], t[1]);
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// 8 elements -> 8 codes for a power-of-two scale: t = x * 2^-e (exact) on pairs.
template <int FMT>
__device__ __forceinline__ uint2 cast_vec_pow2(const uint4& v, float inv) {
    const float2 i2 = make_float2(inv, inv);
    uint32_t c[4];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
        const float2 t = mul2_rn(x, i2);
        c[i] = cvt_pair<FMT>(t.x, t.y);
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// 8 codes -> 8 bf16 of decode(q) * mul, products on pairs.
template <int FMT>
__device__ __forceinline__ uint4 dequant_vec2(const uint2& c, float mul) {
    const float2 m2 = make_float2(mul, mul);
    const float2 a = mul2_rn(decode_pair<FMT>(c.x & 0xFFFFu), m2);
    const float2 b = mul2_rn(decode_pair<FMT>(c.x >> 16), m2);
    const float2 d = mul2_rn(decode_pair<FMT>(c.y & 0xFFFFu), m2);
    const float2 e = mul2_rn(decode_pair<FMT>(c.y >> 16), m2);
    return make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(b.x, b.y), pack_bf16x2(d.x, d.y), pack_bf16x2(e.x, e.y));
}

struct RQParams {
    const uint16_t* x;
    int64_t ld;           // RQ_ROW: row stride (elements)
    int64_t rows, cols;   // RQ_ROW
    int64_t n;            // flat kinds: number of elements (dense tensor)
    uint8_t* q;
    void* scale;
    uint16_t* deq;
    int32_t* status;
    uint32_t* partials;
    int32_t npartials;
    float* ring;
    int32_t ring_len;
    int32_t slot;
    float* pending;
    uint32_t* ticket;
    const float* amax_in;   // RQ_GIVEN
};

// One CTA per row; the row (<= QT * VPT vectors) is held in registers.
template <int FMT, bool DEQ, int VPT, int MINB>
__global__ void __launch_bounds__(QT, MINB) rq_row_kernel(const RQParams p) {
    pdl_launch_dependents();   // a dependent GEMM may start streaming its other operand
    __shared__ uint32_t red[32];
    const int64_t r = blockIdx.x;
    const uint16_t* src = p.x + r * p.ld;
    const int64_t nvec = p.cols / VEC;
    uint4 v[VPT];
    uint32_t m2 = 0;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
        const int64_t k = threadIdx.x + (int64_t)QT * j;
        v[j] = k < nvec ? ld_v4_stream(src + k * VEC) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < VPT; ++j) m2 = bmax_abs_bf16x2(m2, vec_amax2_bf(v[j]));
    uint32_t m = block_max_u32(hmax_pair(m2 & 0x7FFF7FFFu), red);
    if (m >= 0x7F80u) {
        if (threadIdx.x == 0) report_status(p.status, FP8_ERR_NONFINITE);
        m = 0x7F7Fu;
    }
    const RcpScale op = rcp_scale_from_amax_bits<FMT>(m);
    if (threadIdx.x == 0) reinterpret_cast<float*>(p.scale)[r] = op.s;
    uint8_t* dst = p.q + r * p.cols;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
        const int64_t k = threadIdx.x + (int64_t)QT * j;
        if (k < nvec) {
            const uint2 cq = cast_vec_rcp<FMT>(v[j], op);
            *reinterpret_cast<uint2*>(dst + k * VEC) = cq;
            if (DEQ) st_v4_stream(p.deq + r * p.cols + k * VEC, dequant_vec2<FMT>(cq, op.s));
        }
    }
}

// 1x128 / MX32 blocks of a dense tensor: each CTA takes QT * VPT consecutive vectors;
// for a fixed j the vectors of one block sit in G consecutive lanes.
template <int FMT, bool DEQ, int KIND, int VPT>
__global__ void __launch_bounds__(QT, 8) rq_block_kernel(const RQParams p) {
    pdl_launch_dependents();   // a dependent GEMM may start streaming its other operand
    constexpr int G = KIND == RQ_B128 ? 16 : 4;
    const int64_t e0 = (int64_t)blockIdx.x * QT * VPT * VEC;
    uint4 v[VPT];
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
        const int64_t off = e0 + (int64_t)(threadIdx.x + QT * j) * VEC;
        v[j] = off < p.n ? ld_v4_stream(p.x + off) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
        uint32_t m = hmax_pair(vec_amax2_bf(v[j]) & 0x7FFF7FFFu);
#pragma unroll
        for (int o = G / 2; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        const int vec = threadIdx.x + QT * j;
        const int64_t off = e0 + (int64_t)vec * VEC;
        if (off >= p.n) continue;
        if (m >= 0x7F80u) {
            report_status(p.status, FP8_ERR_NONFINITE);
            m = 0x7F7Fu;
        }
        uint2 cq;
        float dmul;
        if (KIND == RQ_B128) {
            const RcpScale op = rcp_scale_from_amax_bits<FMT>(m);
            if ((vec & (G - 1)) == 0) reinterpret_cast<float*>(p.scale)[off / 128] = op.s;
            cq = cast_vec_rcp<FMT>(v[j], op);
            dmul = op.s;
        } else {
            const int e = mx_exponent(m);
            if ((vec & (G - 1)) == 0) reinterpret_cast<uint8_t*>(p.scale)[off / 32] = (uint8_t)(e + 127);
            cq = cast_vec_pow2<FMT>(v[j], exp2i(-e));
            dmul = exp2i(e);
        }
        *reinterpret_cast<uint2*>(p.q + off) = cq;
        if (DEQ) st_v4_stream(p.deq + off, dequant_vec2<FMT>(cq, dmul));
    }
}

// Per-tensor phase 1: U independent loads in flight per thread.
template <int U>
__global__ void __launch_bounds__(QT, 8) rq_amax_kernel(const RQParams p) {
    pdl_launch_dependents();   // a dependent GEMM may start streaming its other operand
    __shared__ uint32_t red[32];
    const int64_t nvec = p.n / VEC;
    uint32_t m2 = 0;
    const int64_t stride = (int64_t)gridDim.x * QT;
    int64_t v = (int64_t)blockIdx.x * QT + threadIdx.x;
    for (; v + (U - 1) * stride < nvec; v += U * stride) {
        uint4 a[U];
#pragma unroll
        for (int u = 0; u < U; ++u) a[u] = ld_v4(p.x + (v + u * stride) * VEC);
#pragma unroll
        for (int u = 0; u < U; ++u) m2 = bmax_abs_bf16x2(m2, vec_amax2_bf(a[u]));
    }
    for (; v < nvec; v += stride) m2 = bmax_abs_bf16x2(m2, vec_amax2_bf(ld_v4(p.x + v * VEC)));
    const uint32_t m = block_max_u32(hmax_pair(m2 & 0x7FFF7FFFu), red);
    if (threadIdx.x == 0) p.partials[blockIdx.x] = m;
}

// Per-tensor phase 2 (RQ_CAST) or the delayed single pass (RQ_DELAYED).
// (The delayed and given-amax kinds also carry the overflow-safe cast: 5 CTAs/SM
// leave them 48 registers.)
template <int FMT, bool DEQ, int KIND, int U>
__global__ void __launch_bounds__(QT, KIND == RQ_CAST ? 6 : 5) rq_tensor_kernel(const RQParams p) {
    pdl_launch_dependents();   // a dependent GEMM may start streaming its other operand
    __shared__ uint32_t red[32];
    uint32_t src = 0;
    if (KIND == RQ_CAST) {
        for (int i = threadIdx.x; i < p.npartials; i += QT) src = max(src, p.partials[i]);
    } else if (KIND == RQ_DELAYED) {
        for (int i = threadIdx.x; i < p.ring_len; i += QT) src = max(src, __float_as_uint(p.ring[i]));
    }
    if (KIND != RQ_GIVEN) src = block_max_u32(src, red);
    float amax;
    bool finite_in = true;     // step 0 of a delayed history records only a finite amax
    if (KIND == RQ_CAST) {
        if (src >= 0x7F80u) {
            if (blockIdx.x == 0 && threadIdx.x == 0) report_status(p.status, FP8_ERR_NONFINITE);
            src = 0x7F7Fu;
            finite_in = false;
        }
        amax = bf16bits_to_float(src);
    } else if (KIND == RQ_DELAYED) {
        amax = __uint_as_float(src);
    } else {
        amax = given_amax(p.amax_in, p.status);
    }
    const float s = scale_from_amax<FMT>(amax);
    const RcpScale op{s, __frcp_rn(s)};
    // With a scale not derived from this input (history, caller), x * (1/s) can
    // overflow fp32; the corrected reciprocal path is exact as long as it does not.
    // Vectors whose |x| stays below 2^127 * s (as a bf16 pattern, rounded down)
    // take it; the rest take the overflow-safe path.
    const uint32_t fast_lim = min(__float_as_uint(__fmul_rn(s, 1.7014118e38f)) >> 16, 0x7F7Fu);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        reinterpret_cast<float*>(p.scale)[0] = s;
        if (KIND == RQ_CAST && p.ring != nullptr && finite_in) p.ring[p.slot] = amax;
    }
    const int64_t nvec = p.n / VEC;
    const int64_t stride = (int64_t)gridDim.x * QT;
    uint32_t m2 = 0;
    auto vec_of = [&](int64_t t) -> int64_t { return KIND == RQ_CAST ? nvec - 1 - t : t; };
    auto emit = [&](int64_t vv, const uint4& a) {
        uint2 cq;
        if (KIND == RQ_DELAYED || KIND == RQ_GIVEN) {
            const uint32_t va = vec_amax2_bf(a);
            m2 = bmax_abs_bf16x2(m2, va);
            cq = hmax_pair(va & 0x7FFF7FFFu) <= fast_lim ? cast_vec_rcp<FMT>(a, op) : cast_vec_rcp_guarded<FMT>(a, op);
        } else {
            cq = cast_vec_rcp<FMT>(a, op);
        }
        __stcs(reinterpret_cast<uint2*>(p.q + vv * VEC), cq);   // evict-first: keep X in L2 for the pass
        if (DEQ) st_v4_stream(p.deq + vv * VEC, dequant_vec2<FMT>(cq, s));
    };
    int64_t t = (int64_t)blockIdx.x * QT + threadIdx.x;
    for (; t + (U - 1) * stride < nvec; t += U * stride) {
        uint4 a[U];
#pragma unroll
        for (int u = 0; u < U; ++u) a[u] = ld_v4(p.x + vec_of(t + u * stride) * VEC);
#pragma unroll
        for (int u = 0; u < U; ++u) emit(vec_of(t + u * stride), a[u]);
    }
    for (; t < nvec; t += stride) emit(vec_of(t), ld_v4(p.x + vec_of(t) * VEC));
    if (KIND == RQ_GIVEN) {
        const uint32_t m = block_max_u32(hmax_pair(m2 & 0x7FFF7FFFu), red);
        if (threadIdx.x == 0 && m >= 0x7F80u) report_status(p.status, FP8_ERR_NONFINITE);
    }
    if (KIND == RQ_DELAYED) {
        const uint32_t m = block_max_u32(hmax_pair(m2 & 0x7FFF7FFFu), red);
        if (threadIdx.x == 0) {
            if (m >= 0x7F80u) report_status(p.status, FP8_ERR_NONFINITE);
            // amax >= 0, so the fp32 bit pattern orders like the value
            atomicMax(reinterpret_cast<uint32_t*>(p.pending), m << 16);
            __threadfence();
            const uint32_t ticket = atomicAdd(p.ticket, 1u);
            if (ticket == gridDim.x - 1) {
                // every CTA read the ring before taking its ticket; a step that saw a
                // NaN/Inf records nothing (its slot keeps the old amax), so one bad step
                // cannot set the scale of the next h steps
                __threadfence();
                const uint32_t a_t = atomicOr(reinterpret_cast<uint32_t*>(p.pending), 0u);
                if (a_t < 0x7F800000u) p.ring[p.slot] = __uint_as_float(a_t);
                *reinterpret_cast<volatile uint32_t*>(p.pending) = 0u;
                *reinterpret_cast<volatile uint32_t*>(p.ticket) = 0u;
            }
        }
    }
}

// Per-tensor current scaling of a small dense tensor (<= 1024 * SMALL_VPT vectors) in
// one CTA: the whole tensor stays in registers through the block-wide amax and the
// cast, so the two launches of the large-tensor path become one.  Same arithmetic
// as rq_amax_kernel + rq_tensor_kernel<RQ_CAST> (codes and scale bit for bit).
constexpr int SMALL_VPT = 8;
constexpr int SMALL_THREADS = 1024;

template <int FMT, bool DEQ>
__global__ void __launch_bounds__(SMALL_THREADS, 1) rq_small_tensor_kernel(const RQParams p) {
    pdl_launch_dependents();   // a dependent GEMM may start streaming its other operand
    __shared__ uint32_t red[32];
    const int64_t nvec = p.n / VEC;
    uint4 v[SMALL_VPT];
    uint32_t m2 = 0;
#pragma unroll
    for (int j = 0; j < SMALL_VPT; ++j) {
        const int64_t k = threadIdx.x + (int64_t)SMALL_THREADS * j;
        v[j] = k < nvec ? ld_v4(p.x + k * VEC) : make_uint4(0, 0, 0, 0);
        m2 = bmax_abs_bf16x2(m2, vec_amax2_bf(v[j]));
    }
    uint32_t m = block_max_u32(hmax_pair(m2 & 0x7FFF7FFFu), red);
    const bool finite_in = m < 0x7F80u;
    if (!finite_in) {
        if (threadIdx.x == 0) report_status(p.status, FP8_ERR_NONFINITE);
        m = 0x7F7Fu;
    }
    const float amax = bf16bits_to_float(m);
    const RcpScale op = rcp_scale_from_amax_bits<FMT>(m);
    if (threadIdx.x == 0) {
        reinterpret_cast<float*>(p.scale)[0] = op.s;
        if (p.ring != nullptr && finite_in) p.ring[p.slot] = amax;   // delayed scaling, step 0
    }
#pragma unroll
    for (int j = 0; j < SMALL_VPT; ++j) {
        const int64_t k = threadIdx.x + (int64_t)SMALL_THREADS * j;
        if (k < nvec) {
            const uint2 cq = cast_vec_rcp<FMT>(v[j], op);
            *reinterpret_cast<uint2*>(p.q + k * VEC) = cq;
            if (DEQ) st_v4_stream(p.deq + k * VEC, dequant_vec2<FMT>(cq, op.s));
        }
    }
}

// ================================================================ per-tensor in one launch
// Current per-tensor scaling needs the whole tensor's a_max before the first code can be
// written ([FFS] "Current Scaling": the amax sits on the critical path).  The two-pass
// kernels above read X twice.  This kernel runs one CTA per SM, all resident at once (a
// cooperative launch), in two phases around one grid-wide exchange of the amax:
//   own   each CTA owns one contiguous piece of X at the front of the tensor: the first
//         PT_HELD_BYTES of it are bulk-copied into shared memory, the next (up to
//         PT_THREADS * PT_REG_VEC vectors) loaded into registers, the rest (up to
//         PT_THREADS * PT_TMEM_VEC vectors) loaded and stored into tensor memory (all
//         512 columns; warp w owns a 128-column group of its lane quarter w % 4); all
//         three stay on chip across the exchange;
//   spill the rest of X, in chunks of PT_SLOT_BYTES dealt round-robin to the CTAs
//         (chunk c to CTA c mod G, so every CTA's share is spread over the whole tensor),
//         streamed through a ring of shared-memory slots filled by bulk copies (many
//         bytes in flight, no registers): for its amax in phase 1, and again, from the
//         last chunk back (the ones the L2 cache still holds), for the cast in phase 2.
// The exchange: every CTA writes its amax into its own slot of the workspace, tagged
// with this call's number, and reads all the slots back (a bounded wait).  The codes
// are those of rq_amax + rq_tensor<CAST> bit for bit: the same integer max over |bf16|
// patterns and the same cast.
//
// The call number: the workspace keeps a 32-bit counter E.  Every CTA reads E before it
// writes its slot, and CTA 0 stores E + 1 only after it has seen every slot, i.e. after
// every CTA has read E; the slots of call E + 1 carry the tag E + 1, so the slots of an
// earlier call (tag <= E) are never taken for this one, whatever the workspace held
// before (a stale or uninitialised slot would also have to match a 16-bit check of its
// tag and CTA).  CUDA-graph replays advance E the same way.
constexpr int PT_THREADS = 512;
constexpr int PT_REG_VEC = 20;                      // 16-byte vectors per thread kept in registers
constexpr uint32_t PT_HELD_BYTES = 96 * 1024;       // bytes per CTA kept in shared memory
constexpr int PT_HELD_CHUNKS = 6;                   // its bulk copies (one mbarrier each)
constexpr int PT_RING = 4;                          // spill ring slots
constexpr uint32_t PT_SLOT_BYTES = 24 * 1024;       // bytes per slot: 3 vectors per thread
constexpr int64_t PT_SLOT_VEC = PT_SLOT_BYTES / 16;
constexpr int PT_TMEM_VEC = 32;                      // 16-byte vectors per thread kept in tensor memory
constexpr int PT_TMEM_BATCH = 4;                     // vectors a thread moves per tcgen05.st / ld
constexpr uint32_t PT_TMEM_COLS = 512;               // all of TMEM: 128 lanes x 512 columns = 256 KB
constexpr int64_t PT_OWN_VEC = PT_HELD_BYTES / 16 + (int64_t)PT_THREADS * (PT_REG_VEC + PT_TMEM_VEC);
constexpr uint32_t PT_DYN_SMEM = PT_HELD_BYTES + PT_RING * PT_SLOT_BYTES + 8 * (PT_HELD_CHUNKS + PT_RING);
constexpr int64_t PT_MIN_ELEMS = (int64_t)16 << 20; // smaller tensors: the two-pass kernels (L2 holds X)

struct PTParams {
    const uint16_t* x;
    int64_t nvec;                  // 16-byte vectors in X
    uint8_t* q;
    float* scale;
    uint16_t* deq;
    int32_t* status;
    uint32_t* epoch;               // workspace: the call counter E
    unsigned long long* slots;     // workspace: one tagged amax per CTA
    float* ring;                   // delayed scaling, step 0: ring[slot] = amax (nullable)
    int32_t slot;
    uint64_t wait_ns;              // limit of the exchange wait
};

__device__ __forceinline__ uint32_t pt_check(uint32_t tag, uint32_t cta) {
    return ((tag * 0x9E3779B1u) ^ (cta * 0x85EBCA77u) ^ 0xA5A5u) >> 16;
}

// A wait for bulk copies this CTA issued (hardware completion; bounded, not cut short).
__device__ __forceinline__ bool pt_wait_copy(uint64_t* bar, uint32_t parity, int32_t* status) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer() - t0 > 2000000000ull) {
            report_status(status, FP8_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

template <int FMT, bool DEQ>
__global__ void __launch_bounds__(PT_THREADS, 1) rq_persist_kernel(const PTParams p) {
    extern __shared__ __align__(1024) uint8_t pt_smem[];
    uint8_t* held = pt_smem;
    uint8_t* ring = pt_smem + PT_HELD_BYTES;
    uint64_t* hbar = reinterpret_cast<uint64_t*>(pt_smem + PT_HELD_BYTES + PT_RING * PT_SLOT_BYTES);
    uint64_t* rbar = hbar + PT_HELD_CHUNKS;
    __shared__ uint32_t red[32];
    __shared__ uint32_t s_epoch;
    __shared__ uint32_t s_tmem;
    const int t = threadIdx.x;
    const int64_t G = gridDim.x, b = blockIdx.x;
    // this CTA's own piece [v0, v1): held part [v0, r0), registers [r0, r1), tensor memory
    // [r1, v1); thread t's j-th vector of the last two is r0 + t + PT_THREADS j (r1 + ...)
    const int64_t v0 = min(p.nvec, b * PT_OWN_VEC), v1 = min(p.nvec, v0 + PT_OWN_VEC);
    const int64_t n_held = min(v1 - v0, (int64_t)(PT_HELD_BYTES / 16));
    const int64_t r0 = v0 + n_held;
    const int64_t r1 = min(v1, r0 + (int64_t)PT_THREADS * PT_REG_VEC);
    const int warp = t >> 5;
    // this thread's TMEM words: lane (warp % 4) * 32 + lane, columns from (warp / 4) * 128
    const uint32_t tm_off = ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(warp >> 2) * 128u;
    // the spill: everything past the own pieces, in chunks of PT_SLOT_VEC vectors
    const int64_t sp0 = min(p.nvec, G * PT_OWN_VEC);
    const int64_t nsc = (p.nvec - sp0 + PT_SLOT_VEC - 1) / PT_SLOT_VEC;
    const uint4* xv = reinterpret_cast<const uint4*>(p.x);
    const uint32_t held_bytes = (uint32_t)(n_held * 16);
    const uint32_t hchunk = (held_bytes / PT_HELD_CHUNKS + 15u) & ~15u;   // a multiple of 16
    const int nhc = hchunk ? (int)((held_bytes + hchunk - 1) / hchunk) : 0;
    // this CTA's spill chunks: c = b + i G in phase 1 (i < nb), then c = nsc - 1 - b - i G
    // in phase 2; ring use j < 2 nb goes to slot j % PT_RING with parity (j / PT_RING) & 1
    const int64_t nb = b < nsc ? (nsc - 1 - b) / G + 1 : 0;
    auto chunk_of = [&](int64_t j) { return j < nb ? b + j * G : (nsc - 1 - b) - (j - nb) * G; };

    if (t == 0) {
        s_epoch = *reinterpret_cast<volatile uint32_t*>(p.epoch);   // read before this CTA arrives
        for (int c = 0; c < PT_HELD_CHUNKS + PT_RING; ++c) ptx::mbar_init(&hbar[c], 1);
        ptx::fence_mbar_init();
    }
    if (warp == 0) {                                   // one CTA per SM: all of TMEM is free
        ptx::tmem_alloc(&s_tmem, PT_TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();                                   // the barriers, s_epoch and s_tmem are set
    ptx::tc_fence_after();
    const uint32_t tmem = s_tmem + tm_off;
    const uint32_t tag = s_epoch + 1u;
    const uint64_t pol_keep = ptx::createpolicy_evict_last(), pol_drop = ptx::createpolicy_evict_first();
    // one thread: copy the chunk of ring use j into its slot (the first read keeps its
    // lines in L2 for the re-read; the re-read drops them)
    auto issue = [&](int64_t j) {
        const int64_t cv0 = sp0 + chunk_of(j) * PT_SLOT_VEC;
        const uint32_t bytes = (uint32_t)(min(PT_SLOT_VEC, p.nvec - cv0) * 16);
        const int sl = (int)(j % PT_RING);
        ptx::mbar_arrive_expect_tx(&rbar[sl], bytes);
        ptx::bulk_load_1d_hint(ring + sl * PT_SLOT_BYTES, xv + cv0, bytes, &rbar[sl], j < nb ? pol_keep : pol_drop);
    };
    // ring uses [j0, j1): fn(slot vectors, first vector index of the chunk, count); the
    // copy of use j + PT_RING (up to jmax) goes out as soon as slot j is free
    auto run_ring = [&](int64_t j0, int64_t j1, int64_t jmax, auto&& fn) -> bool {
        bool ok = true;
        for (int64_t j = j0; j < j1; ++j) {
            const int sl = (int)(j % PT_RING);
            ok &= pt_wait_copy(&rbar[sl], (uint32_t)((j / PT_RING) & 1), p.status);
            const int64_t cv0 = sp0 + chunk_of(j) * PT_SLOT_VEC;
            fn(reinterpret_cast<const uint4*>(ring + sl * PT_SLOT_BYTES), cv0, min(PT_SLOT_VEC, p.nvec - cv0));
            __syncthreads();                           // every thread is done with slot sl
            if (t == 0 && j + PT_RING < jmax) issue(j + PT_RING);
        }
        return ok;
    };
    if (t == 0) {
        for (int c = 0; c < nhc; ++c) {
            const uint32_t off = (uint32_t)c * hchunk;
            const uint32_t nbytes = min(hchunk, held_bytes - off);
            ptx::mbar_arrive_expect_tx(&hbar[c], nbytes);
            ptx::bulk_load_1d_hint(held + off, reinterpret_cast<const uint8_t*>(xv + v0) + off, nbytes, &hbar[c],
                                   pol_drop);
        }
        for (int64_t j = 0; j < min(2 * nb, (int64_t)PT_RING); ++j) issue(j);
    }
    // ---- phase 1: a_max of the registers, the TMEM part, the spill chunks and the held part
    uint4 reg[PT_REG_VEC];
#pragma unroll
    for (int j = 0; j < PT_REG_VEC; ++j) {
        const int64_t k = r0 + t + (int64_t)PT_THREADS * j;
        reg[j] = k < r1 ? ld_v4_stream(xv + k) : make_uint4(0, 0, 0, 0);
    }
    uint32_t m2 = 0;
    // the TMEM part, PT_TMEM_BATCH vectors at a time: batch i's loads go out one spill
    // chunk before its max and its store, so that their latency overlaps the stream
    constexpr int NTB = PT_TMEM_VEC / PT_TMEM_BATCH;
    uint4 tb[PT_TMEM_BATCH];
    int next_tb = 0;
    auto load_tb = [&](int i) {
#pragma unroll
        for (int u = 0; u < PT_TMEM_BATCH; ++u) {
            const int64_t k = r1 + t + (int64_t)PT_THREADS * (i * PT_TMEM_BATCH + u);
            tb[u] = k < v1 ? ld_v4_stream(xv + k) : make_uint4(0, 0, 0, 0);
        }
    };
    auto store_tb = [&](int i) {                       // warp-collective
        uint32_t w[16];
#pragma unroll
        for (int u = 0; u < PT_TMEM_BATCH; ++u) {
            m2 = bmax_abs_bf16x2(m2, vec_amax2_bf(tb[u]));
            w[4 * u] = tb[u].x;
            w[4 * u + 1] = tb[u].y;
            w[4 * u + 2] = tb[u].z;
            w[4 * u + 3] = tb[u].w;
        }
        ptx::tmem_st_32x32b_x16(tmem + (uint32_t)(16 * i), w);
    };
    load_tb(0);
    // phase 1's ring also sends out phase 2's first copies as the ring empties
    bool fail = !run_ring(0, nb, 2 * nb, [&](const uint4* sv, int64_t, int64_t nv) {
        for (int64_t k = t; k < nv; k += PT_THREADS) m2 = bmax_abs_bf16x2(m2, vec_amax2_bf(sv[k]));
        if (next_tb < NTB) {
            store_tb(next_tb);
            if (++next_tb < NTB) load_tb(next_tb);
        }
    });
    while (next_tb < NTB) {
        store_tb(next_tb);
        if (++next_tb < NTB) load_tb(next_tb);
    }
    ptx::tmem_st_wait();
#pragma unroll
    for (int j = 0; j < PT_REG_VEC; ++j) m2 = bmax_abs_bf16x2(m2, vec_amax2_bf(reg[j]));
    for (int c = 0; c < nhc; ++c) fail |= !pt_wait_copy(&hbar[c], 0, p.status);
    for (int64_t k = t; k < n_held; k += PT_THREADS)
        m2 = bmax_abs_bf16x2(m2, vec_amax2_bf(*reinterpret_cast<const uint4*>(held + k * 16)));
    const uint32_t m_cta = block_max_u32(hmax_pair(m2 & 0x7FFF7FFFu), red);
    // ---- the exchange
    if (t == 0) {
        const unsigned long long word = ((unsigned long long)tag << 32) |
                                        ((unsigned long long)pt_check(tag, (uint32_t)b) << 16) | m_cta;
        atomicExch(p.slots + b, word);
    }
    uint32_t gm = 0;
    if (!fail) {
        const uint64_t t0 = ptx::globaltimer();
        for (int64_t i = t; i < G && !fail; i += PT_THREADS) {
            const volatile unsigned long long* sp = p.slots + i;
            while (true) {
                const unsigned long long w = *sp;
                if ((uint32_t)(w >> 32) == tag && (uint32_t)((w >> 16) & 0xFFFFu) == pt_check(tag, (uint32_t)i)) {
                    gm = max(gm, (uint32_t)(w & 0xFFFFu));
                    break;
                }
                if (ptx::globaltimer() - t0 > p.wait_ns) {
                    report_status(p.status, FP8_ERR_TIMEOUT);
                    fail = true;
                    break;
                }
                __nanosleep(64);
            }
        }
    }
    fail = __syncthreads_or(fail) != 0;
    // CTA 0 advances the call counter once its wait has ended, whether or not the exchange
    // completed: on success every CTA has read E by then (it arrived).  (After a time-out a
    // CTA that had not even started could still read the new value; the workspace is then
    // undefined until the caller zeroes it, which the interface states.)
    if (b == 0 && t == 0) *reinterpret_cast<volatile uint32_t*>(p.epoch) = tag;
    if (fail) {
        // outputs unspecified; phase 2's copies already issued must land before the CTA exits
        if (t == 0)
            for (int64_t j = nb; j < min(2 * nb, nb + (int64_t)PT_RING); ++j)
                pt_wait_copy(&rbar[j % PT_RING], (uint32_t)((j / PT_RING) & 1), p.status);
        ptx::tc_fence_before();
        __syncthreads();                               // every thread's TMEM stores are complete
        if (warp == 0) ptx::tmem_dealloc(s_tmem, PT_TMEM_COLS);
        return;
    }
    gm = block_max_u32(gm, red);
    const bool finite_in = gm < 0x7F80u;
    if (!finite_in) {
        if (b == 0 && t == 0) report_status(p.status, FP8_ERR_NONFINITE);
        gm = 0x7F7Fu;                                  // keep the scale finite; outputs unspecified
    }
    const RcpScale op = rcp_scale_from_amax_bits<FMT>(gm);
    if (b == 0 && t == 0) {
        p.scale[0] = op.s;
        if (p.ring != nullptr && finite_in) p.ring[p.slot] = bf16bits_to_float(gm);
    }
    pdl_launch_dependents();                           // a dependent GEMM may start streaming its other operand
    // ---- phase 2: the cast of the spill (from the last chunk back), registers, held part
    auto emit = [&](int64_t k, const uint4& a) {
        const uint2 cq = cast_vec_rcp<FMT>(a, op);
        __stcs(reinterpret_cast<uint2*>(p.q) + k, cq);
        if (DEQ) st_v4_stream(p.deq + k * VEC, dequant_vec2<FMT>(cq, op.s));
    };
    run_ring(nb, 2 * nb, 2 * nb, [&](const uint4* sv, int64_t cv0, int64_t nv) {
        for (int64_t k = t; k < nv; k += PT_THREADS) emit(cv0 + k, sv[k]);
    });
#pragma unroll
    for (int j = 0; j < PT_REG_VEC; ++j) {
        const int64_t k = r0 + t + (int64_t)PT_THREADS * j;
        if (k < r1) emit(k, reg[j]);
    }
    for (int i = 0; i < NTB; ++i) {                    // warp-collective loads
        uint32_t w[16];
        ptx::tmem_ld_32x32b_x16(tmem + (uint32_t)(16 * i), w);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < PT_TMEM_BATCH; ++u) {
            const int64_t k = r1 + t + (int64_t)PT_THREADS * (i * PT_TMEM_BATCH + u);
            if (k < v1) emit(k, make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]));
        }
    }
    for (int64_t k = t; k < n_held; k += PT_THREADS) emit(v0 + k, *reinterpret_cast<const uint4*>(held + k * 16));
    ptx::tc_fence_before();
    __syncthreads();                                   // every thread's TMEM loads are complete
    if (warp == 0) ptx::tmem_dealloc(s_tmem, PT_TMEM_COLS);
}

// ================================================================ launchers
static int sm_count_cached() {
    static int cache[kDeviceCacheSlots];   // per device
    const int ds = device_slot();
    if (ds >= 0 && cache[ds] > 0) return cache[ds];
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    if (ds >= 0) cache[ds] = n;
    return n;
}

int32_t amax_partials_count() { return 148 * 8; }

// Grid for the streaming per-tensor kernels: at most amax_partials_count() CTAs.
static dim3 tensor_grid(int64_t nrows, int64_t nvec) {
    const int64_t cap = std::min<int64_t>(amax_partials_count(), (int64_t)sm_count_cached() * 8);
    int64_t gx = std::max<int64_t>(1, std::min<int64_t>((nvec + QT - 1) / QT, cap));
    int64_t gy = std::max<int64_t>(1, std::min<int64_t>(nrows, cap / gx));
    gy = std::min<int64_t>(gy, 65535);
    return dim3((unsigned)gx, (unsigned)gy);
}

template <int FMT, bool DEQ>
static void launch_cast_tensor(const QuantArgs& a, int src, dim3 grid, int npart, float* ring, int32_t len,
                               int32_t slot, float* pending, uint32_t* ticket, int64_t nrows, int64_t nvec,
                               int64_t ld, cudaStream_t st) {
    if (src == SRC_PARTIALS)
        cast_tensor_kernel<FMT, DEQ, SRC_PARTIALS><<<grid, QT, 0, st>>>(
            a.x, nrows, nvec, ld, a.partials, npart, ring, len, slot, pending, ticket, a.q,
            (float*)a.scale, a.deq, a.status);
    else if (src == SRC_GIVEN)
        cast_tensor_kernel<FMT, DEQ, SRC_GIVEN><<<grid, QT, 0, st>>>(
            a.x, nrows, nvec, ld, nullptr, 0, const_cast<float*>(a.amax_in), 1, 0, nullptr, nullptr, a.q,
            (float*)a.scale, a.deq, a.status);
    else
        cast_tensor_kernel<FMT, DEQ, SRC_RING><<<grid, QT, 0, st>>>(
            a.x, nrows, nvec, ld, a.partials, npart, ring, len, slot, pending, ticket, a.q,
            (float*)a.scale, a.deq, a.status);
}

static int64_t rq_grid_cap() { return std::min<int64_t>(amax_partials_count(), (int64_t)sm_count_cached() * 8); }

// Cooperative launch of rq_persist_kernel (all CTAs resident at once), one grid per
// SM count times the CTAs that fit per SM (known per device, at most one slot per CTA).
// `launched` stays false when the kernel cannot run here (the caller then takes the
// two-pass kernels).
template <int FMT, bool DEQ>
static cudaError_t launch_persist(const PTParams& pt, cudaStream_t st, bool& launched) {
    static int ctas_per_sm[kDeviceCacheSlots];      // 0: unknown, -1: not usable, else CTAs per SM
    const int ds = device_slot();
    int per_sm = ds >= 0 ? ctas_per_sm[ds] : 0;
    const size_t dyn = PT_DYN_SMEM;
    if (per_sm == 0) {
        int coop = 0, dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
        int n = 0;
        if (coop &&
            cudaFuncSetAttribute(rq_persist_kernel<FMT, DEQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)dyn) == cudaSuccess &&
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, rq_persist_kernel<FMT, DEQ>, PT_THREADS, dyn) ==
                cudaSuccess &&
            n > 0)
            per_sm = n;
        else
            per_sm = -1;
        cudaGetLastError();                          // a refused attribute is not this call's error
        if (ds >= 0) ctas_per_sm[ds] = per_sm;
    }
    if (per_sm <= 0) return cudaSuccess;
    const int64_t grid = std::min<int64_t>((int64_t)per_sm * sm_count_cached(), 1184);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(PT_THREADS);
    cfg.dynamicSmemBytes = dyn;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, rq_persist_kernel<FMT, DEQ>, pt);
    launched = e == cudaSuccess;
    if (!launched) cudaGetLastError();               // e.g. the device is shared: the two passes run instead
    return cudaSuccess;
}

template <int FMT, bool DEQ>
static cudaError_t rq_tensor_t(const QuantArgs& a, cudaStream_t st) {
    RQParams p{};
    p.x = a.x;
    p.n = a.rows * a.cols;
    p.q = a.q;
    p.scale = a.scale;
    p.deq = a.deq;
    p.status = a.status;
    p.partials = a.partials;
    p.ring = a.hist_ring;
    p.ring_len = a.hist_len;
    p.slot = a.hist_ring ? (int32_t)(a.hist_step % a.hist_len) : 0;
    p.pending = a.hist_pending;
    p.ticket = a.hist_ticket;
    const int64_t nvec = p.n / VEC;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(rq_grid_cap(), (nvec + QT - 1) / QT));
    if (a.hist_ring != nullptr && a.hist_step > 0) {
        rq_tensor_kernel<FMT, DEQ, RQ_DELAYED, 4><<<(unsigned)grid, QT, 0, st>>>(p);
        return cudaGetLastError();
    }
    if (nvec <= (int64_t)SMALL_THREADS * SMALL_VPT) {
        rq_small_tensor_kernel<FMT, DEQ><<<1, SMALL_THREADS, 0, st>>>(p);
        return cudaGetLastError();
    }
    if (p.n >= PT_MIN_ELEMS && (reinterpret_cast<uintptr_t>(a.partials) & 7u) == 0) {
        PTParams pt{};
        pt.x = a.x;
        pt.nvec = nvec;
        pt.q = a.q;
        pt.scale = static_cast<float*>(a.scale);
        pt.deq = a.deq;
        pt.status = a.status;
        pt.epoch = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(a.partials) + kEpochOffset);
        pt.slots = reinterpret_cast<unsigned long long*>(reinterpret_cast<uint8_t*>(a.partials) + kSlotsOffset);
        pt.ring = a.hist_ring;
        pt.slot = p.slot;
        pt.wait_ns = wait_limit_ns();
        bool launched = false;
        launch_persist<FMT, DEQ>(pt, st, launched);
        if (launched) return cudaSuccess;
    }
    rq_amax_kernel<8><<<(unsigned)grid, QT, 0, st>>>(p);
    p.npartials = (int32_t)grid;
    rq_tensor_kernel<FMT, DEQ, RQ_CAST, 4><<<(unsigned)grid, QT, 0, st>>>(p);
    return cudaGetLastError();
}

// Per-tensor current scaling (two launches) or one delayed step.
cudaError_t launch_quantize_tensor(const QuantArgs& a, cudaStream_t st) {
    const bool dense = a.ld == a.cols;
    if (dense && a.rows > 0 && a.cols > 0) {
        if (a.fmt == FP8_E4M3) return a.deq ? rq_tensor_t<FP8_E4M3, true>(a, st) : rq_tensor_t<FP8_E4M3, false>(a, st);
        return a.deq ? rq_tensor_t<FP8_E5M2, true>(a, st) : rq_tensor_t<FP8_E5M2, false>(a, st);
    }
    const int64_t nrows = dense ? (a.rows > 0 ? 1 : 0) : a.rows;
    const int64_t nvec = dense ? a.rows * a.cols / VEC : a.cols / VEC;
    dim3 grid = tensor_grid(std::max<int64_t>(nrows, 1), std::max<int64_t>(nvec, 1));
    const int npart = (int)(grid.x * grid.y);
    const bool delayed_t = a.hist_ring != nullptr && a.hist_step > 0;
    const int32_t slot = a.hist_ring ? (int32_t)(a.hist_step % a.hist_len) : 0;
    if (!delayed_t)
        amax_partials_kernel<<<grid, QT, 0, st>>>(a.x, nrows, nvec, a.ld, a.partials);
    const int src = delayed_t ? SRC_RING : SRC_PARTIALS;
    const bool deq = a.deq != nullptr;
    if (a.fmt == FP8_E4M3) {
        if (deq) launch_cast_tensor<FP8_E4M3, true>(a, src, grid, npart, a.hist_ring, a.hist_len, slot, a.hist_pending, a.hist_ticket, nrows, nvec, a.ld, st);
        else     launch_cast_tensor<FP8_E4M3, false>(a, src, grid, npart, a.hist_ring, a.hist_len, slot, a.hist_pending, a.hist_ticket, nrows, nvec, a.ld, st);
    } else {
        if (deq) launch_cast_tensor<FP8_E5M2, true>(a, src, grid, npart, a.hist_ring, a.hist_len, slot, a.hist_pending, a.hist_ticket, nrows, nvec, a.ld, st);
        else     launch_cast_tensor<FP8_E5M2, false>(a, src, grid, npart, a.hist_ring, a.hist_len, slot, a.hist_pending, a.hist_ticket, nrows, nvec, a.ld, st);
    }
    return cudaGetLastError();
}

// fp8_amax: one CTA folds the phase-1 partials into the fp32 amax.
__global__ void __launch_bounds__(QT) amax_finalize_kernel(const uint32_t* __restrict__ partials, int32_t n,
                                                           float* __restrict__ out, int32_t* status) {
    __shared__ uint32_t red[32];
    uint32_t m = 0;
    for (int i = threadIdx.x; i < n; i += QT) m = max(m, partials[i]);
    m = block_max_u32(m, red);
    if (threadIdx.x == 0) {
        if (m >= 0x7F80u) report_status(status, FP8_ERR_NONFINITE);
        *out = bf16bits_to_float(m);
    }
}

cudaError_t launch_amax(const QuantArgs& a, float* out, cudaStream_t st) {
    if (a.rows == 0 || a.cols == 0) return cudaMemsetAsync(out, 0, sizeof(float), st);
    int32_t npart;
    if (a.ld == a.cols) {
        RQParams p{};
        p.x = a.x;
        p.n = a.rows * a.cols;
        p.partials = a.partials;
        const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(rq_grid_cap(), (p.n / VEC + QT - 1) / QT));
        rq_amax_kernel<8><<<(unsigned)grid, QT, 0, st>>>(p);
        npart = (int32_t)grid;
    } else {
        const dim3 grid = tensor_grid(a.rows, a.cols / VEC);
        amax_partials_kernel<<<grid, QT, 0, st>>>(a.x, a.rows, a.cols / VEC, a.ld, a.partials);
        npart = (int32_t)(grid.x * grid.y);
    }
    amax_finalize_kernel<<<1, QT, 0, st>>>(a.partials, npart, out, a.status);
    return cudaGetLastError();
}

template <int FMT, bool DEQ>
static cudaError_t quantize_given_t(const QuantArgs& a, cudaStream_t st) {
    if (a.ld == a.cols || a.rows == 0 || a.cols == 0) {
        RQParams p{};
        p.x = a.x;
        p.n = a.rows * a.cols;
        p.q = a.q;
        p.scale = a.scale;
        p.deq = a.deq;
        p.status = a.status;
        p.amax_in = a.amax_in;
        const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(rq_grid_cap(), (p.n / VEC + QT - 1) / QT));
        rq_tensor_kernel<FMT, DEQ, RQ_GIVEN, 4><<<(unsigned)grid, QT, 0, st>>>(p);
        return cudaGetLastError();
    }
    const dim3 grid = tensor_grid(a.rows, a.cols / VEC);
    launch_cast_tensor<FMT, DEQ>(a, SRC_GIVEN, grid, 0, nullptr, 0, 0, nullptr, nullptr, a.rows, a.cols / VEC, a.ld,
                                 st);
    return cudaGetLastError();
}

// Per-tensor cast with a caller's amax (empty tensors still write the scale).
cudaError_t launch_quantize_given(const QuantArgs& a, cudaStream_t st) {
    if (a.fmt == FP8_E4M3) return a.deq ? quantize_given_t<FP8_E4M3, true>(a, st) : quantize_given_t<FP8_E4M3, false>(a, st);
    return a.deq ? quantize_given_t<FP8_E5M2, true>(a, st) : quantize_given_t<FP8_E5M2, false>(a, st);
}

template <int FMT, bool DEQ, int G, int U, bool MX>
static void launch_segment(const QuantArgs& a, int32_t seg_vec, cudaStream_t st) {
    const int64_t seg_elems = (int64_t)seg_vec * VEC;
    const int64_t nspr = (a.cols + seg_elems - 1) / seg_elems;
    const int64_t nseg = a.rows * nspr;
    if (nseg == 0) return;
    const bool flat = a.ld == a.cols && a.cols % seg_elems == 0;
    const int64_t groups_needed = nseg;
    const int64_t cap = (int64_t)sm_count_cached() * 8;
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((groups_needed * G + QT - 1) / QT, cap * 16));
    if (flat)
        quant_segment_kernel<FMT, DEQ, G, U, MX, true><<<(unsigned)blocks, QT, 0, st>>>(
            a.x, a.rows, a.cols, a.ld, seg_vec, nspr, nseg, a.q, a.scale, a.deq, a.status);
    else
        quant_segment_kernel<FMT, DEQ, G, U, MX, false><<<(unsigned)blocks, QT, 0, st>>>(
            a.x, a.rows, a.cols, a.ld, seg_vec, nspr, nseg, a.q, a.scale, a.deq, a.status);
}

template <int FMT, bool DEQ>
static cudaError_t quantize_grouped_t(const QuantArgs& a, cudaStream_t st) {
    // register-resident kernels for the shapes they cover (rows of 1-16 Ki elements;
    // dense tensors for the 1x128 and MX32 blocks)
    {
        RQParams p{};
        p.x = a.x;
        p.ld = a.ld;
        p.rows = a.rows;
        p.cols = a.cols;
        p.n = a.rows * a.cols;
        p.q = a.q;
        p.scale = a.scale;
        p.deq = a.deq;
        p.status = a.status;
        if (a.mode == FP8_SCALE_ROW && a.cols >= 1024 && a.cols <= 16384 && a.rows > 0 && a.rows < ((int64_t)1 << 31)) {
            const unsigned g = (unsigned)a.rows;
            const int64_t vpt = (a.cols / VEC + QT - 1) / QT;
            if (vpt <= 1)      rq_row_kernel<FMT, DEQ, 1, 8><<<g, QT, 0, st>>>(p);
            else if (vpt <= 2) rq_row_kernel<FMT, DEQ, 2, 8><<<g, QT, 0, st>>>(p);
            else if (vpt <= 4) rq_row_kernel<FMT, DEQ, 4, 8><<<g, QT, 0, st>>>(p);
            else               rq_row_kernel<FMT, DEQ, 8, 4><<<g, QT, 0, st>>>(p);
            return cudaGetLastError();
        }
        const bool dense = a.ld == a.cols && a.rows > 0 && a.cols > 0;
        if (dense && ((a.mode == FP8_SCALE_BLOCK_1x128 && a.cols % 128 == 0) || a.mode == FP8_SCALE_MX32)) {
            const int64_t per_cta = (int64_t)QT * 4 * VEC;
            const int64_t grid = (p.n + per_cta - 1) / per_cta;
            if (grid < ((int64_t)1 << 31)) {
                if (a.mode == FP8_SCALE_MX32) rq_block_kernel<FMT, DEQ, RQ_MX, 4><<<(unsigned)grid, QT, 0, st>>>(p);
                else                          rq_block_kernel<FMT, DEQ, RQ_B128, 4><<<(unsigned)grid, QT, 0, st>>>(p);
                return cudaGetLastError();
            }
        }
    }
    switch (a.mode) {
    case FP8_SCALE_ROW: {
        const int64_t nvec = a.cols / VEC;
        if (nvec <= 32 * 8) {
            // short rows: a warp (or less) per row
            if (nvec <= 4 * 4)       launch_segment<FMT, DEQ, 4, 4, false>(a, (int32_t)nvec, st);
            else if (nvec <= 16 * 4) launch_segment<FMT, DEQ, 16, 4, false>(a, (int32_t)nvec, st);
            else                     launch_segment<FMT, DEQ, 32, 8, false>(a, (int32_t)nvec, st);
        } else {
            const int64_t blocks = std::min<int64_t>(a.rows, (int64_t)1 << 30);
            if (nvec <= QT * 4)
                quant_row_kernel<FMT, DEQ, 4><<<(unsigned)blocks, QT, 0, st>>>(a.x, a.rows, a.cols, a.ld, a.q, (float*)a.scale, a.deq, a.status);
            else
                quant_row_kernel<FMT, DEQ, 8><<<(unsigned)blocks, QT, 0, st>>>(a.x, a.rows, a.cols, a.ld, a.q, (float*)a.scale, a.deq, a.status);
        }
        break;
    }
    case FP8_SCALE_BLOCK_1x128:
        launch_segment<FMT, DEQ, 4, 4, false>(a, 16, st);
        break;
    case FP8_SCALE_MX32:
        launch_segment<FMT, DEQ, 4, 1, true>(a, 4, st);
        break;
    case FP8_SCALE_BLOCK_128x128: {
        dim3 grid((unsigned)((a.cols + 127) / 128), (unsigned)((a.rows + 127) / 128));
        if (grid.x && grid.y)
            quant_block128_kernel<FMT, DEQ><<<grid, QT, 0, st>>>(a.x, a.rows, a.cols, a.ld, a.q, (float*)a.scale, a.deq, a.status);
        break;
    }
    default:
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_quantize_grouped(const QuantArgs& a, cudaStream_t st) {
    const bool deq = a.deq != nullptr;
    if (a.fmt == FP8_E4M3) return deq ? quantize_grouped_t<FP8_E4M3, true>(a, st) : quantize_grouped_t<FP8_E4M3, false>(a, st);
    if (a.mode == FP8_SCALE_MX32) return cudaErrorInvalidValue;
    return deq ? quantize_grouped_t<FP8_E5M2, true>(a, st) : quantize_grouped_t<FP8_E5M2, false>(a, st);
}

// Scales of empty inputs: amax = 0 gives the floor scale (MX: byte 0).
__global__ void fill_floor_scale_kernel(float* s, int64_t n, float v) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) s[i] = v;
}

cudaError_t launch_fill_scale(float* s, int64_t n, float v, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const int64_t blocks = std::min<int64_t>((n + 255) / 256, 1024);
    fill_floor_scale_kernel<<<(unsigned)blocks, 256, 0, st>>>(s, n, v);
    return cudaGetLastError();
}

}  // namespace fp8b
