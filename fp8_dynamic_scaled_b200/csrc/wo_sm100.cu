// wo_sm100.cu -- weight-only FP8 linear for few tokens (M <= 64), sm_100a.
//
//   Y[m, n] = bf16( s_w[n] sum_k x[m,k] decode(w[n,k]) ),  X bf16, W FP8 codes,
//   s_w per tensor or per output channel
//
// [FFS] "FP8 formats, scaling and LLM inference", section "Weight-only FP8 与 W8A8
// FP8": the weight is stored in FP8 and the activation stays BF16; the kernel reads
// FP8 and converts it, and the gain is the weight's memory and bandwidth.  tcgen05
// multiplies BF16 by BF16 (kind::f16) but not BF16 by FP8, so:
//   - the weight streams exactly as in the W8A8 decode kernel (decode_sm100.cu):
//     one contiguous range of W rows per SM in 16-row units, chunks of <= 128 rows,
//     stages of 3 K blocks loaded as 64-/16-row boxes issued row group by row group;
//     every FP8 code is read from HBM once;
//   - eight converter warps turn each 128-row x 64-element half of a K block into
//     BF16 (exact: every E4M3 and E5M2 value is a BF16 value) and store it straight into
//     tensor memory (tcgen05.st: TMEM lane = weight row, two BF16 per 32-bit column),
//     into a ring of WO_SLOTS 32-column slots, so the BF16 weight never goes through
//     shared memory;
//   - the MMA warp issues tcgen05.mma kind::f16 with the weight as A read from TMEM
//     (M = 128 rows) and the tokens as B (N = M rounded up to 16, X tiles loaded by TMA
//     as BF16 into shared memory), FP32 accumulators double-buffered in TMEM across
//     chunks;
//   - the epilogue warp of a TMEM lane quarter owns 32 weight rows and writes
//     bf16(acc * s_w[n]) for every token.
// Every wait is bounded as in the other kernels.
//
// Up to WG_MAX_TOKENS (3) tokens the product is a matrix-vector one whose bound is
// the weight's bytes, and a tcgen05.mma with N = 16 (the smallest at M = 128) moves only
// 2 KB of FP8 weight per instruction as BF16; there fp8_wo_gemv_kernel does the
// contraction on the CUDA cores instead: W streamed once with 16-byte loads, codes
// decoded in registers, FP32 accumulation on packed f32x2 FMAs.
#include "gemm_common.cuh"

namespace fp8b {

constexpr int WO_UNIT = 16;                          // rows of W per work unit
constexpr int WO_TILE = 128;                         // rows of W per MMA
constexpr int WO_KBS = 3;                            // K blocks (128 codes) per stage
constexpr int WO_MAX_STAGES = 4;
constexpr int WO_SLOTS = 8;                          // BF16 weight ring in TMEM (32 columns a slot)
constexpr uint32_t WO_ACC_COLS = 128;                // TMEM columns 0-127: two accumulators of <= 64
constexpr uint32_t WO_TMEM_COLS = 512;
constexpr int WO_CONV_WARPS = 8, WO_EPI_WARPS = 4;
constexpr int WO_FIRST_CONV = 2, WO_FIRST_EPI = WO_FIRST_CONV + WO_CONV_WARPS;
constexpr int WO_THREADS = 32 * (WO_FIRST_EPI + WO_EPI_WARPS);     // 448
constexpr uint32_t WO_W8_BYTES = WO_TILE * BK;       // 16 KB: FP8 codes of one K block
constexpr uint32_t WO_BAR_BYTES = 1024;
constexpr uint32_t WO_SMEM = 227 * 1024;

struct WoParams {
    int32_t units;          // ceil(N / 16)
    int32_t nt;             // tokens per MMA: M rounded up to 16
    int32_t stages;
    uint32_t stage_bytes;   // WO_KBS * (WO_W8_BYTES + 2 * nt * 128)
};

struct WoRange {
    int32_t u0, cnt, nch;
};

__device__ __forceinline__ WoRange wo_range(int32_t units, int32_t c, int32_t ctas) {
    const int32_t base = units / ctas, extra = units % ctas;
    WoRange r;
    r.u0 = c * base + min(c, extra);
    r.cnt = base + (c < extra ? 1 : 0);
    r.nch = (r.cnt + 7) / 8;
    return r;
}

__device__ __forceinline__ void wo_chunk(const WoRange& r, int32_t j, int32_t& n0, int32_t& w) {
    const int32_t ua = r.u0 + 8 * j;
    const int32_t ub = min(ua + 8, r.u0 + r.cnt);
    n0 = ua * WO_UNIT;
    w = (ub - ua) * WO_UNIT;
}

// 16 FP8 codes (one 16-byte chunk) -> 16 BF16 values packed two per word (element 2i
// in the low half of word i), exact.
template <int WFMT>
__device__ __forceinline__ void codes16_to_bf16(const uint4& c, uint32_t* o) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = decode_pair<WFMT>(w[i] & 0xFFFFu);
        const float2 b = decode_pair<WFMT>(w[i] >> 16);
        o[2 * i] = pack_bf16x2(a.x, a.y);
        o[2 * i + 1] = pack_bf16x2(b.x, b.y);
    }
}

template <int WFMT>
__global__ void __launch_bounds__(WO_THREADS, 1)
fp8_wo_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW64,
              const __grid_constant__ CUtensorMap tmW16, const GemmParams p, const WoParams d) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + WO_MAX_STAGES;
    uint64_t* afull = empty + WO_MAX_STAGES;           // a BF16 slot is written (converters)
    uint64_t* aempty = afull + WO_SLOTS;               // its MMAs are done (commit)
    uint64_t* tfull = aempty + WO_SLOTS;
    uint64_t* tempty = tfull + 2;
    uint64_t* teardown = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(teardown + 1);
    volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);
    // stage s: FP8 W of WO_KBS K blocks (16 KB each), then X as 2 * WO_KBS BF16 halves
    uint8_t* stages = smem + WO_BAR_BYTES;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const WoRange range = wo_range(d.units, blockIdx.x, gridDim.x);
    const int32_t S = d.stages;
    const int32_t nkc = (p.num_kb + WO_KBS - 1) / WO_KBS;     // stages per chunk
    const uint32_t x_off = WO_KBS * WO_W8_BYTES;
    const uint32_t x_half = (uint32_t)d.nt * 128;               // bytes of one X half tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(&full[s], 1);
            // the stage is free once the converters have read its W codes and the MMAs
            // its X tiles
            ptx::mbar_init(&empty[s], WO_CONV_WARPS + 1);
        }
        for (int t = 0; t < WO_SLOTS; ++t) {
            ptx::mbar_init(&afull[t], WO_CONV_WARPS);
            ptx::mbar_init(&aempty[t], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], WO_EPI_WARPS);
        }
        ptx::mbar_init(teardown, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmX);
        ptx::prefetch_tmap(&tmW64);
        ptx::prefetch_tmap(&tmW16);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, WO_TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            IssuedLoads loads;
            for (int32_t j = 0; j < range.nch && ok; ++j) {
                int32_t n0, w;
                wo_chunk(range, j, n0, w);
                for (int32_t kc = 0; kc < nkc; ++kc) {
                    const int32_t kb0 = kc * WO_KBS;
                    const int32_t kbs = min(WO_KBS, p.num_kb - kb0);
                    if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status, p.wait_ns)) { ok = false; break; }
                    uint8_t* st = stages + stage * d.stage_bytes;
                    ptx::mbar_arrive_expect_tx(&full[stage], (uint32_t)kbs * ((uint32_t)w * BK + 2 * x_half));
                    for (int32_t r = 0; r < w;) {
                        const bool big = w - r >= 64;
                        for (int32_t b = 0; b < kbs; ++b)
                            ptx::tma_load_2d(st + b * WO_W8_BYTES + r * BK, big ? &tmW64 : &tmW16, &full[stage],
                                             (kb0 + b) * BK, n0 + r);
                        r += big ? 64 : WO_UNIT;
                    }
                    for (int32_t b = 0; b < kbs; ++b)
                        for (int h = 0; h < 2; ++h)
                            ptx::tma_load_2d(st + x_off + (2 * b + h) * x_half, &tmX, &full[stage],
                                             (kb0 + b) * BK + h * 64, 0);
                    loads.note(stage, phase);
                    if (++stage == (uint32_t)S) { stage = 0; phase ^= 1u; }
                }
            }
            loads.drain(full, p.status);      // loads in flight after an abort
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer: D[n, m] += W_bf16 X^T
        uint32_t stage = 0, phase = 0, acc_it = 0, conv_it = 0;
        bool ok = true;
        const uint32_t s0 = ptx::smem_u32(stages);
        for (int32_t j = 0; j < range.nch && ok; ++j) {
            const uint32_t buf = acc_it & 1u, use = acc_it >> 1;
            if (!wait_bounded(&tempty[buf], (use & 1u) ^ 1u, abort_flag, p.status, p.wait_ns)) { ok = false; break; }
            ptx::tc_fence_after();
            for (int32_t kc = 0; kc < nkc && ok; ++kc) {
                const int32_t kbs = min(WO_KBS, p.num_kb - kc * WO_KBS);
                if (!wait_bounded(&full[stage], phase, abort_flag, p.status, p.wait_ns)) { ok = false; break; }
                const uint32_t sx = s0 + stage * d.stage_bytes + x_off;
                for (int32_t hb = 0; hb < 2 * kbs; ++hb) {
                    const uint32_t t = conv_it % WO_SLOTS, tu = conv_it / WO_SLOTS;
                    if (!wait_bounded(&afull[t], tu & 1u, abort_flag, p.status, p.wait_ns)) { ok = false; break; }
                    ptx::tc_fence_after();
                    if (lane == 0) {
                        const uint32_t a0 = tmem_base + WO_ACC_COLS + t * 32;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {                       // K = 16 BF16 per instruction
                            const uint64_t bd = ptx::sdesc_kmajor_sw128(sx + hb * x_half + k * 32);
                            ptx::mma_f16_ts(tmem_base + buf * 64, a0 + k * 8, bd, p.idesc, (kc | hb | k) != 0);
                        }
                        ptx::mma_commit(&aempty[t]);
                    }
                    __syncwarp();
                    ++conv_it;
                }
                if (!ok) break;
                if (lane == 0) ptx::mma_commit(&empty[stage]);      // its X tiles are read
                __syncwarp();
                if (++stage == (uint32_t)S) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            if (lane == 0) ptx::mma_commit(&tfull[buf]);
            __syncwarp();
            ++acc_it;
        }
        if (lane == 0) {                      // issued MMAs finish before TMEM is freed
            ptx::mma_commit(teardown);
            wait_drain(teardown, 0, p.status);
        }
        __syncwarp();
    } else if (warp < WO_FIRST_EPI) {
        // ------------------------------------------------ converters: FP8 -> BF16 in TMEM
        // warp cw owns the 32 weight rows of its TMEM lane quarter and one 32-value part of
        // each 64-value half K block: 32 codes a thread -> 16 words -> one 16-column store
        const int cw = warp - WO_FIRST_CONV;                 // 0 .. 7
        const int quarter = warp & 3;                        // TMEM lane quarter of this warp
        const int part = cw >> 2;                            // 32-value part of a half K block
        const int row = quarter * 32 + lane;
        const int sw = row & 7;                              // the row's 128-byte swizzle phase
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        uint32_t stage = 0, phase = 0, conv_it = 0;
        bool ok = true;
        for (int32_t j = 0; j < range.nch && ok; ++j) {
            for (int32_t kc = 0; kc < nkc && ok; ++kc) {
                const int32_t kbs = min(WO_KBS, p.num_kb - kc * WO_KBS);
                if (!wait_bounded(&full[stage], phase, abort_flag, p.status, p.wait_ns)) { ok = false; break; }
                const uint8_t* w8 = stages + stage * d.stage_bytes;
                for (int32_t hb = 0; hb < 2 * kbs; ++hb) {
                    const uint32_t t = conv_it % WO_SLOTS, tu = conv_it / WO_SLOTS;
                    if (!wait_bounded(&aempty[t], (tu & 1u) ^ 1u, abort_flag, p.status, p.wait_ns)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const int b = hb >> 1, h = hb & 1;
                    const uint8_t* src = w8 + b * WO_W8_BYTES + row * 128;
                    uint32_t o[16];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int jj = 4 * h + 2 * part + q;          // 16-code chunk of the 128-byte row
                        codes16_to_bf16<WFMT>(*reinterpret_cast<const uint4*>(src + ((jj ^ sw) * 16)), o + 8 * q);
                    }
                    ptx::tmem_st_32x32b_x16(tmem_base + lane_base + WO_ACC_COLS + t * 32 + part * 16, o);
                    ptx::tmem_st_wait();
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&afull[t]);
                    ++conv_it;
                }
                if (!ok) break;
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&empty[stage]);     // its W codes are read
                if (++stage == (uint32_t)S) { stage = 0; phase ^= 1u; }
            }
        }
    } else {
        // ------------------------------------------------ epilogue: lane = weight row
        const int quarter = warp & 3;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        uint32_t acc_it = 0;
        for (int32_t j = 0; j < range.nch; ++j) {
            int32_t n0, w;
            wo_chunk(range, j, n0, w);
            const uint32_t buf = acc_it & 1u, use = acc_it >> 1;
            if (!wait_bounded(&tfull[buf], use & 1u, abort_flag, p.status, p.wait_ns)) break;
            ptx::tc_fence_after();
            const int32_t r = quarter * 32 + lane;
            const int32_t n = n0 + r;
            const bool valid = r < w && n < p.N;
            if (quarter * 32 < w) {                                // warp-uniform
                const float sw = valid ? __ldg(p.sb + (int64_t)n * p.sb_stride) : 0.0f;
                for (int32_t c0 = 0; c0 < p.M; c0 += 16) {
                    uint32_t acc[16];
                    ptx::tmem_ld_32x32b_x16(tmem_base + lane_base + buf * 64 + c0, acc);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int tk = 0; tk < 16; ++tk) {
                        const int32_t m = c0 + tk;
                        if (m < p.M && valid)
                            p.y[(int64_t)m * p.ldy + n] = (uint16_t)(pack_bf16x2(__uint_as_float(acc[tk]) * sw, 0.0f) & 0xFFFFu);
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
            ++acc_it;
        }
    }

    // ------------------------------------------------ teardown
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem_base, WO_TMEM_COLS);
}

template <int WFMT>
static cudaError_t launch_wo_t(const WoArgs& g, cudaStream_t st) {
    GemmParams p{};
    p.wait_ns = wait_limit_ns();
    p.M = (int32_t)g.M;
    p.N = (int32_t)g.N;
    p.K = (int32_t)g.K;
    p.num_kb = (int32_t)((g.K + BK - 1) / BK);
    p.sb = static_cast<const float*>(g.sw);
    p.sb_stride = g.w_row_scales ? 1 : 0;
    p.status = g.status;
    p.y = g.y;
    p.ldy = g.ldy;
    WoParams d{};
    d.nt = (int32_t)((g.M + 15) / 16 * 16);
    d.units = (int32_t)((g.N + WO_UNIT - 1) / WO_UNIT);
    d.stage_bytes = WO_KBS * (WO_W8_BYTES + 2u * (uint32_t)d.nt * 128);
    d.stages = (int32_t)std::min<uint32_t>(WO_MAX_STAGES, (WO_SMEM - 1024 - WO_BAR_BYTES) / d.stage_bytes);
    // BF16 x BF16 (kind::f16: formats 1 = BF16 in bits 7-9 and 10-12), FP32 D, M = 128, N = nt
    p.idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(d.nt >> 3) << 17) | ((uint32_t)(WO_TILE >> 4) << 24);
    CUtensorMap tx, t64, t16;
    if (!make_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.x, (uint64_t)g.K, (uint64_t)g.M, (uint64_t)g.ldx * 2,
                     64, (uint32_t)d.nt, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&t64, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.w, (uint64_t)g.K, (uint64_t)g.N, (uint64_t)g.K, BK, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&t16, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.w, (uint64_t)g.K, (uint64_t)g.N, (uint64_t)g.K, BK, 16,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    static bool attr_done[kDeviceCacheSlots];   // the attribute is set per device
    const int ds = device_slot();
    if (ds < 0 || !attr_done[ds]) {
        cudaError_t e = cudaFuncSetAttribute(fp8_wo_kernel<WFMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)WO_SMEM);
        if (e != cudaSuccess) return e;
        if (ds >= 0) attr_done[ds] = true;
    }
    const uint32_t smem = 1024 + WO_BAR_BYTES + (uint32_t)d.stages * d.stage_bytes;
    const int grid = std::max(1, std::min(d.units, num_sms()));
    fp8_wo_kernel<WFMT><<<grid, WO_THREADS, smem, st>>>(tx, t64, t16, p, d);
    return cudaGetLastError();
}

// ================================================================ matrix-vector path
// A warp owns 8 consecutive weight rows.  Lane l works on rows (l >> 3) and
// (l >> 3) + 4 of them and on the 16-code chunk (l & 7) of every 128-code step, so
// the 8 lanes of a row read one full 128-byte line of it per step and each lane
// converts its X chunk once for two rows.  After the K loop the 8 partial sums of
// a row are added with shuffles and lane (l & 7) == 0 writes bf16(sum * s_w[n]).
// Loads are in bounds by construction: n < N, k0 + 16 <= K (K % 16 == 0), m < M.
constexpr int WG_THREADS = 256;
constexpr int WG_MAX_TOKENS = 3;                        // measured: at 4 tokens the tensor-core kernel ties

template <int MT>
struct WgShape {
    static constexpr int U = MT <= 2 ? 2 : 1;           // 128-code steps in flight per lane (measured)
};

template <int WFMT, int MT>
__global__ void __launch_bounds__(WG_THREADS, 4)
fp8_wo_gemv_kernel(const uint16_t* __restrict__ x, int64_t ldx, const uint8_t* __restrict__ w,
                   const float* __restrict__ sw, int32_t sw_stride, int32_t N, int32_t K,
                   uint16_t* __restrict__ y, int64_t ldy) {
    constexpr int U = WgShape<MT>::U;
    const int lane = threadIdx.x & 31;
    const int sub = lane & 7, slot = lane >> 3;
    const int64_t warp0 = ((int64_t)blockIdx.x * WG_THREADS + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * WG_THREADS) >> 5;
    const int64_t groups = ((int64_t)N + 7) / 8;
    const int32_t steps = (K + 127) / 128;
    for (int64_t g = warp0; g < groups; g += nwarps) {            // warp-uniform
        const int32_t n0 = (int32_t)(g * 8) + slot, n1 = n0 + 4;
        const bool v0 = n0 < N, v1 = n1 < N;
        const uint8_t* w0 = w + (int64_t)(v0 ? n0 : 0) * K;
        const uint8_t* w1 = w + (int64_t)(v1 ? n1 : 0) * K;
        float2 acc[MT][2];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m][0] = acc[m][1] = make_float2(0.0f, 0.0f);
        for (int32_t s = 0; s < steps; s += U) {
            uint4 a[U][2];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t k0 = (int64_t)(s + u) * 128 + sub * 16;
                const bool kin = k0 < K;
                a[u][0] = (kin && v0) ? __ldcs(reinterpret_cast<const uint4*>(w0 + k0)) : make_uint4(0, 0, 0, 0);
                a[u][1] = (kin && v1) ? __ldcs(reinterpret_cast<const uint4*>(w1 + k0)) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t k0 = (int64_t)(s + u) * 128 + sub * 16;
                if (k0 >= K) continue;
                // the chunk in two halves of 8 codes, so that few decoded values are live
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    // codes 8h + 2q and 8h + 2q + 1 -> wf[r][q]
                    float2 wf[2][4];
                    const uint32_t c0[2] = {h ? a[u][0].z : a[u][0].x, h ? a[u][0].w : a[u][0].y};
                    const uint32_t c1[2] = {h ? a[u][1].z : a[u][1].x, h ? a[u][1].w : a[u][1].y};
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        wf[0][2 * i] = decode_pair<WFMT>(c0[i] & 0xFFFFu);
                        wf[0][2 * i + 1] = decode_pair<WFMT>(c0[i] >> 16);
                        wf[1][2 * i] = decode_pair<WFMT>(c1[i] & 0xFFFFu);
                        wf[1][2 * i + 1] = decode_pair<WFMT>(c1[i] >> 16);
                    }
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const uint4 xv4 = __ldg(reinterpret_cast<const uint4*>(x + (int64_t)m * ldx + k0 + 8 * h));
                        const uint32_t xv[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            // bf16 pair -> exact fp32 pair (the even value in the low half)
                            const float2 xf =
                                make_float2(__uint_as_float(xv[q] << 16), __uint_as_float(xv[q] & 0xFFFF0000u));
                            acc[m][0] = ptx::ffma2(xf, wf[0][q], acc[m][0]);
                            acc[m][1] = ptx::ffma2(xf, wf[1][q], acc[m][1]);
                        }
                    }
                }
            }
        }
        const float s0 = v0 ? __ldg(sw + (int64_t)n0 * sw_stride) : 0.0f;
        const float s1 = v1 ? __ldg(sw + (int64_t)n1 * sw_stride) : 0.0f;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float t0 = acc[m][0].x + acc[m][0].y, t1 = acc[m][1].x + acc[m][1].y;
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                t0 += __shfl_xor_sync(0xFFFFFFFFu, t0, o);
                t1 += __shfl_xor_sync(0xFFFFFFFFu, t1, o);
            }
            if (sub == 0) {
                if (v0) y[(int64_t)m * ldy + n0] = (uint16_t)(pack_bf16x2(t0 * s0, 0.0f) & 0xFFFFu);
                if (v1) y[(int64_t)m * ldy + n1] = (uint16_t)(pack_bf16x2(t1 * s1, 0.0f) & 0xFFFFu);
            }
        }
    }
}

template <int WFMT, int MT>
static cudaError_t launch_gemv_t(const WoArgs& g, cudaStream_t st) {
    static int per_sm_of[kDeviceCacheSlots];              // resident CTAs per SM, per device
    const int ds = device_slot();
    int per_sm = ds >= 0 ? per_sm_of[ds] : 0;
    if (per_sm == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fp8_wo_gemv_kernel<WFMT, MT>, WG_THREADS, 0) !=
                cudaSuccess ||
            per_sm <= 0)
            per_sm = 1;
        if (ds >= 0) per_sm_of[ds] = per_sm;
    }
    const int64_t groups = (g.N + 7) / 8;
    const int64_t want = (groups + WG_THREADS / 32 - 1) / (WG_THREADS / 32);      // one row group per warp
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)num_sms() * per_sm));
    fp8_wo_gemv_kernel<WFMT, MT><<<grid, WG_THREADS, 0, st>>>(g.x, g.ldx, g.w, static_cast<const float*>(g.sw),
                                                              g.w_row_scales ? 1 : 0, (int32_t)g.N, (int32_t)g.K,
                                                              g.y, g.ldy);
    return cudaGetLastError();
}

template <int WFMT>
static cudaError_t launch_gemv(const WoArgs& g, cudaStream_t st) {
    static_assert(WG_MAX_TOKENS == 3, "one instantiation per token count");
    switch (g.M) {
        case 1: return launch_gemv_t<WFMT, 1>(g, st);
        case 2: return launch_gemv_t<WFMT, 2>(g, st);
        case 3: return launch_gemv_t<WFMT, 3>(g, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_weight_only(const WoArgs& g, cudaStream_t st) {
    if (g.M <= WG_MAX_TOKENS)
        return g.w_fmt == FP8_E4M3 ? launch_gemv<FP8_E4M3>(g, st) : launch_gemv<FP8_E5M2>(g, st);
    return g.w_fmt == FP8_E4M3 ? launch_wo_t<FP8_E4M3>(g, st) : launch_wo_t<FP8_E5M2>(g, st);
}

}  // namespace fp8b
