// gemm_common.cuh -- pieces shared by the FP8 GEMM kernels of libfp8 (the tiled
// and CTA-pair kernels in gemm_sm100.cu, the weight-streaming kernel in
// decode_sm100.cu): tile constants, kernel parameters, bounded mbarrier waits, the
// epilogue (scales, optional bias / output amax / FP8 output, output staging) and
// the host-side tensor-map helpers.  sm_100a only.
#pragma once

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace fp8b {

constexpr int BM = 128;             // rows of A per tile (TMEM lanes)
constexpr int BN = 256;             // rows of B per tile (TMEM columns)
constexpr int BK = 128;             // K bytes per pipeline stage (one 128-byte swizzle row)
constexpr int UMMA_K = 32;          // K per tcgen05.mma for 8-bit operands
constexpr int STAGES = 4;
constexpr uint32_t A_STAGE_BYTES = BM * BK;   // 16 KB
constexpr uint32_t B_STAGE_BYTES = BN * BK;   // 32 KB
constexpr uint64_t WAIT_TIMEOUT_NS = 4000000000ull;   // 4 s: default limit of a pipeline wait
constexpr uint64_t DRAIN_LIMIT_NS = 2000000000ull;    // 2 s: limit of a wait for hardware completion


struct GemmParams {
    int32_t M, N, K;
    int32_t num_m, num_n, num_kb;
    int32_t m_fastest;
    int32_t group;          // tiles of the fast dimension per raster group
    // ROWSCALE: element scale = sa[m * sa_stride] * sb[n * sb_stride]
    const float* sa;
    const float* sb;
    int32_t sa_stride, sb_stride;
    // BLOCK: sa [M][num_kb], sb [ceil(N/128)][num_kb];  MX: E8M0 bytes [rows][K/32]
    const uint8_t* sfa;
    const uint8_t* sfb;
    uint32_t idesc;
    int32_t* status;
    // output written with plain stores when it cannot be described to TMA
    // (row stride not a multiple of 16 bytes, or a base address off 16 bytes)
    uint16_t* y;
    int64_t ldy;
    int32_t y_direct;
    int32_t y_vec;          // y rows start 16-byte aligned (ldy % 8 == 0, aligned base)
    int32_t sb_vec;         // per-row b scales start 16-byte aligned
    // optional epilogue (fp8_epilogue_t); ext != 0 when any option is set
    int32_t ext;
    int32_t write_y;        // 0: no bf16 Y (FP8 output only)
    const uint16_t* bias;   // bf16 [N], 16-byte aligned, or null
    uint32_t* amax;         // fp32 bit pattern folded with atomicMax, or null
    uint8_t* yq;            // FP8 codes [M, ldq], or null
    const float* yq_scale;
    int64_t ldq;
    int32_t yq_fmt;
    int32_t yq_vec;         // yq rows start 16-byte aligned
    // launched as the programmatic dependent of the kernel that produced A (and only A);
    // every kernel waits (pdl_wait) before it reads A or the scales
    int32_t pdl;
    uint64_t wait_ns;       // limit of each pipeline wait (wait_limit_ns() at launch)
};

// ---------------------------------------------------------------- bounded waits
// A pipeline wait: gives up when another warp of the CTA has raised the abort flag, or
// after limit_ns, when it raises the flag itself and reports FP8_ERR_TIMEOUT.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int32_t* abort_flag,
                                             int32_t* status, uint64_t limit_ns) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer();
    if (limit_ns < 1000000ull) {
        // a short limit (the failure-path tests): each test suspends the thread for at most
        // 100 ns, so that the limit is checked well before a slow phase could complete
        while (true) {
            if (ptx::mbar_try_wait_hint(bar, parity, 100u)) return true;
            if (*abort_flag) return false;
            if (ptx::globaltimer() - t0 > limit_ns) {
                *abort_flag = 1;
                report_status(status, FP8_ERR_TIMEOUT);
                return false;
            }
        }
    }
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (ptx::globaltimer() - t0 > limit_ns) {
            *abort_flag = 1;
            report_status(status, FP8_ERR_TIMEOUT);
            return false;
        }
    }
}

// A wait for a phase that the hardware completes by itself (the bytes of a TMA load
// this CTA issued, a tcgen05.commit of MMAs it issued).  Unlike a pipeline wait it
// ignores the abort flag: an aborting CTA must not release its shared memory or its
// TMEM while a copy or an MMA still writes or reads them.  Still bounded (2 s), so
// that nothing can hold the GPU; on expiry it reports FP8_ERR_TIMEOUT and returns.
__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity, int32_t* status) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer() - t0 > DRAIN_LIMIT_NS) {
            report_status(status, FP8_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// The TMA loads a producer thread has issued: per ring stage, whether any was issued
// and the phase parity of the last one.  The last load of a stage completes the
// phase of that parity on the stage's full barrier (earlier ones completed before the
// stage was refilled), so waiting for those phases waits for every load in flight.
struct IssuedLoads {
    uint32_t issued = 0, parity = 0;
    __device__ __forceinline__ void note(uint32_t stage, uint32_t phase) {
        issued |= 1u << stage;
        parity = (parity & ~(1u << stage)) | ((phase & 1u) << stage);
    }
    // Before the CTA may exit: every issued load has landed.
    __device__ __forceinline__ void drain(uint64_t* full, int32_t* status) const {
        for (uint32_t s = 0; s < 32; ++s)
            if ((issued >> s) & 1u) wait_drain(&full[s], (parity >> s) & 1u, status);
    }
};

// Write 32 bf16 (16 packed words) of one row into a 32x32 staging tile laid out
// for the 64-byte TMA swizzle: 16-byte chunk j of row r sits at chunk j ^ ((r>>1)&3).
__device__ __forceinline__ void stage_row_sw64(uint8_t* buf, int r, const uint32_t (&w)[16]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int jj = j ^ ((r >> 1) & 3);
        *reinterpret_cast<uint4*>(buf + r * 64 + jj * 16) = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
    }
}

// Store a 32-row x 32-column bf16 chunk held one row per lane (columns >= n_lim are
// not written by the plain-store path; the TMA path clips at the tensor edge).
__device__ __forceinline__ void store_chunk(const CUtensorMap* tmY, uint8_t* buf, const uint32_t (&w)[16],
                                            int32_t x, int32_t y, int lane, const GemmParams& p, int32_t n_lim) {
    if (p.y_direct) {
        const int32_t row = y + lane;
        if (row < p.M) {
            uint16_t* dst = p.y + (int64_t)row * p.ldy;
            if (p.y_vec && n_lim - x >= 32 && (x & 7) == 0) {
                uint4* d4 = reinterpret_cast<uint4*>(dst + x);
#pragma unroll
                for (int q = 0; q < 4; ++q) d4[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                return;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int32_t n = x + 2 * j;
                if (n < n_lim) dst[n] = (uint16_t)(w[j] & 0xFFFFu);
                if (n + 1 < n_lim) dst[n + 1] = (uint16_t)(w[j] >> 16);
            }
        }
        return;
    }
    stage_row_sw64(buf, lane, w);
    ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        ptx::tma_store_2d(tmY, buf, x, y);
        ptx::bulk_commit();
    }
}

// ---------------------------------------------------------------- optional epilogue
// Per-lane state of the fp8_epilogue_t options: the running |y| maximum and the
// constants of the FP8 output cast y_q = RNE(clip(y / s_y)).
struct EpiState {
    uint32_t amax2;        // packed |bf16| maxima (sign bits meaningless)
    float2 s2, nr2;        // s_y and -1/s_y in both lanes
    uint32_t lo2, hi2;     // clip bounds of y as packed bf16 pairs
    bool yq_ok;
};

__device__ __forceinline__ EpiState epi_init(const GemmParams& p) {
    EpiState e;
    e.amax2 = 0;
    e.s2 = e.nr2 = make_float2(0.0f, 0.0f);
    e.lo2 = e.hi2 = 0;
    e.yq_ok = false;
    if (p.ext && p.yq) {
        const float s = __ldg(p.yq_scale);
        // s and 1/s both normal: 2^-126 <= s <= 2^126
        e.yq_ok = s >= 1.17549435e-38f && s <= 8.5070592e37f;
        if (!e.yq_ok && (threadIdx.x & 31) == 0) report_status(p.status, FP8_ERR_INVALID_ARG);
        if (e.yq_ok) {
            const float r = __frcp_rn(s);
            e.s2 = make_float2(s, s);
            e.nr2 = make_float2(-r, -r);
            // y / s_y is computed as a reciprocal with one Markstein correction, exact
            // (as IEEE division) while y * (1/s_y) stays finite.  |y| is first clipped
            // to the largest bf16 <= 2^127 s_y: anything beyond saturates either way.
            const uint32_t lim = min(__float_as_uint(__fmul_rn(s, 1.7014118e38f)) >> 16, 0x7F7Fu);
            e.hi2 = lim | (lim << 16);
            e.lo2 = e.hi2 | 0x80008000u;
        }
    }
    return e;
}

// The options on 32 columns [n0, n0 + 32) of one output row held by this lane (only
// columns below n_lim exist):
// f[] are the scaled fp32 accumulators.  Adds the bias, rounds to bf16 (w, for the
// Y store), folds |y| into the running maximum and writes the FP8 output codes.
__device__ __forceinline__ void epi_chunk(const GemmParams& p, EpiState& es, float (&f)[32], int32_t n0,
                                          int32_t n_lim, int32_t row, uint32_t (&w)[16]) {
    if (p.bias) {
        if (n0 + 32 <= n_lim) {
            const uint4* b4 = reinterpret_cast<const uint4*>(p.bias + n0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 b = __ldg(b4 + q);
                const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 s = add2_rn(make_float2(f[8 * q + 2 * i], f[8 * q + 2 * i + 1]),
                                             make_float2(bf16_lo(bw[i]), bf16_hi(bw[i])));
                    f[8 * q + 2 * i] = s.x;
                    f[8 * q + 2 * i + 1] = s.y;
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float b = n0 + j < n_lim ? bf16bits_to_float(__ldg(p.bias + n0 + j)) : 0.0f;
                f[j] = __fadd_rn(f[j], b);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(f[2 * j], f[2 * j + 1]);
    if (row >= p.M) return;
    if (p.amax) {
#pragma unroll
        for (int j = 0; j < 16; ++j) es.amax2 = bmax_abs_bf16x2(es.amax2, w[j]);
    }
    if (es.yq_ok) {
        uint32_t c[8];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            // on -y with -1/s_y: q = RN(y r), e = -(y - q s) exactly, t = RN(q + (y - q s) r);
            // keeps the sign of a zero y
            const uint32_t wn = clamp_bf16x2(w[j], es.lo2, es.hi2) ^ 0x80008000u;
            const float2 nx = make_float2(__uint_as_float(wn << 16), __uint_as_float(wn & 0xFFFF0000u));
            const float2 q = mul2_rn(nx, es.nr2);
            const float2 e = fma2_rn(q, es.s2, nx);
            const float2 t = fma2_rn(e, es.nr2, q);
            const uint32_t code = p.yq_fmt == FP8_E4M3 ? cvt_pair<FP8_E4M3>(t.x, t.y) : cvt_pair<FP8_E5M2>(t.x, t.y);
            c[j / 2] = (j & 1) ? (c[j / 2] | (code << 16)) : code;
        }
        uint8_t* dst = p.yq + (int64_t)row * p.ldq + n0;
        if (n0 + 32 <= n_lim && p.yq_vec) {
            reinterpret_cast<uint4*>(dst)[0] = make_uint4(c[0], c[1], c[2], c[3]);
            reinterpret_cast<uint4*>(dst)[1] = make_uint4(c[4], c[5], c[6], c[7]);
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (n0 + j < n_lim) dst[j] = (uint8_t)(c[j / 4] >> (8 * (j & 3)));
        }
    }
}

// End of a warp's epilogue: fold its |y| maximum into the caller's amax.
__device__ __forceinline__ void epi_flush(const GemmParams& p, const EpiState& es, int lane) {
    if (!p.amax) return;
    const uint32_t m = __reduce_max_sync(0xffffffffu, hmax_pair(es.amax2 & 0x7FFF7FFFu));
    // |y| >= 0: the fp32 bit pattern (bf16 pattern << 16) orders like the value
    if (lane == 0 && m != 0) atomicMax(p.amax, m << 16);
}

// Per-tensor / per-row scales on 32 accumulator columns of one row:
// y = acc * (s_a[m] * s_b[n]), then the plain bf16 rounding or the options.
template <bool EXT>
__device__ __forceinline__ void rowscale_chunk(const GemmParams& p, EpiState& es, const uint32_t (&r)[32], float sx,
                                               int32_t n0, int32_t n_lim, int32_t row, uint32_t (&w)[16]) {
    if constexpr (!EXT) {
        if (n0 + 32 <= n_lim && (p.sb_stride == 0 || p.sb_vec)) {
            // whole chunk: the 32 channel scales as eight 16-byte loads (the same for
            // every lane), products on f32x2 pairs; the same roundings as below
            const float2 sx2 = make_float2(sx, sx);
            const float4* sb4 = reinterpret_cast<const float4*>(p.sb + n0);
            const float sb0 = p.sb_stride == 0 ? __ldg(p.sb) : 0.0f;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 b = p.sb_stride == 0 ? make_float4(sb0, sb0, sb0, sb0) : __ldg(sb4 + q);
                const float2 s01 = mul2_rn(sx2, make_float2(b.x, b.y));
                const float2 s23 = mul2_rn(sx2, make_float2(b.z, b.w));
                const float2 v01 = mul2_rn(make_float2(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1])), s01);
                const float2 v23 = mul2_rn(make_float2(__uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3])), s23);
                w[2 * q] = pack_bf16x2(v01.x, v01.y);
                w[2 * q + 1] = pack_bf16x2(v23.x, v23.y);
            }
            return;
        }
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
            const int32_t n = n0 + j;
            const float s0 = n < n_lim ? sx * __ldg(p.sb + (int64_t)n * p.sb_stride) : 0.0f;
            const float s1 = n + 1 < n_lim ? sx * __ldg(p.sb + (int64_t)(n + 1) * p.sb_stride) : 0.0f;
            w[j / 2] = pack_bf16x2(__uint_as_float(r[j]) * s0, __uint_as_float(r[j + 1]) * s1);
        }
    } else {
        // columns at or past n_lim are zero (their accumulators may hold anything)
        float f[32];
        if (n0 + 32 <= n_lim && (p.sb_stride == 0 || p.sb_vec)) {
            const float2 sx2 = make_float2(sx, sx);
            const float4* sb4 = reinterpret_cast<const float4*>(p.sb + n0);
            const float sb0 = p.sb_stride == 0 ? __ldg(p.sb) : 0.0f;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 b = p.sb_stride == 0 ? make_float4(sb0, sb0, sb0, sb0) : __ldg(sb4 + q);
                const float2 v01 = mul2_rn(make_float2(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1])),
                                           mul2_rn(sx2, make_float2(b.x, b.y)));
                const float2 v23 = mul2_rn(make_float2(__uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3])),
                                           mul2_rn(sx2, make_float2(b.z, b.w)));
                f[4 * q] = v01.x;
                f[4 * q + 1] = v01.y;
                f[4 * q + 2] = v23.x;
                f[4 * q + 3] = v23.y;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int32_t n = n0 + j;
                f[j] = n < n_lim ? __uint_as_float(r[j]) * (sx * __ldg(p.sb + (int64_t)n * p.sb_stride)) : 0.0f;
            }
        }
        epi_chunk(p, es, f, n0, n_lim, row, w);
    }
}

// Tile raster: the operand with the smaller footprint is walked fastest, in groups
// of `group` tiles whose panels fit comfortably in L2; within a group the fast index
// varies fastest and the group sweeps the whole slow dimension before the next group.
__device__ __forceinline__ void tile_coords(const GemmParams& p, int32_t t, int32_t& mb, int32_t& nb) {
    const int32_t nfast = p.m_fastest ? p.num_m : p.num_n;
    const int32_t nslow = p.m_fastest ? p.num_n : p.num_m;
    const int32_t per_group = p.group * nslow;
    const int32_t g = t / per_group;
    const int32_t rem = t - g * per_group;
    const int32_t width = min(p.group, nfast - g * p.group);
    const int32_t fast = g * p.group + rem % width;
    const int32_t slow = rem / width;
    if (p.m_fastest) { mb = fast; nb = slow; }
    else             { nb = fast; mb = slow; }
}

// ================================================================ host side
// Raster group for a given row-tile height (see tile_coords).
inline int32_t raster_group(int64_t nfast, int64_t panel_bytes) {
    int64_t grp = std::max<int64_t>(1, (int64_t)36 * 1024 * 1024 / std::max<int64_t>(panel_bytes, 1));
    if (grp >= nfast) return (int32_t)std::max<int64_t>(nfast, 1);
    const int64_t ngroups = (nfast + grp - 1) / grp;
    return (int32_t)std::max<int64_t>((nfast + ngroups - 1) / ngroups, 1);
}


typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// The last maps this host thread encoded, direct-mapped by their arguments: a call that
// passes the same buffers and shapes again (a serving loop) copies the 128-byte map
// instead of encoding it anew.  A map depends only on these arguments.
struct MapKey {
    uint64_t base, inner, outer, row_bytes;
    uint32_t box_inner, box_outer, dt, sw;
};
struct MapSlot {
    MapKey key;
    CUtensorMap map;
    bool valid;
};
constexpr int kMapCacheSlots = 32;

static bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                        uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    static thread_local MapSlot cache[kMapCacheSlots];
    MapKey key;
    std::memset(&key, 0, sizeof(key));
    key.base = reinterpret_cast<uint64_t>(base);
    key.inner = inner;
    key.outer = outer;
    key.row_bytes = row_bytes;
    key.box_inner = box_inner;
    key.box_outer = box_outer;
    key.dt = (uint32_t)dt;
    key.sw = (uint32_t)sw;
    uint64_t h = key.base ^ (inner * 0x9E3779B97F4A7C15ull) ^ (outer * 0xC2B2AE3D27D4EB4Full) ^
                 ((uint64_t)box_outer << 17) ^ ((uint64_t)box_inner << 29) ^ ((uint64_t)key.dt << 41) ^ row_bytes;
    h ^= h >> 29;
    MapSlot& slot = cache[(h ^ (h >> 7)) % kMapCacheSlots];
    if (slot.valid && std::memcmp(&slot.key, &key, sizeof(key)) == 0) {
        *m = slot.map;
        return true;
    }
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    slot.key = key;
    slot.map = *m;
    slot.valid = true;
    return true;
}

static int num_sms() {
    static int cache[kDeviceCacheSlots];
    const int ds = device_slot();
    if (ds >= 0 && cache[ds] > 0) return cache[ds];
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    if (ds >= 0) cache[ds] = n;
    return n;
}

// The weight-streaming kernel for few-token calls (decode_sm100.cu): per-tensor /
// per-row scales, M <= D_MAX_TOKENS.
constexpr int64_t D_MAX_TOKENS = 64;
cudaError_t launch_decode(const GemmArgs& g, const GemmParams& p, cudaStream_t st);

}  // namespace fp8b
