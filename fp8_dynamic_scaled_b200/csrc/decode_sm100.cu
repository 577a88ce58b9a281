// decode_sm100.cu -- FP8 scaled GEMM for few-token calls (M <= 64), sm_100a.
//
//   Y[m, n] = bf16( s_a[m] s_b[n] sum_k a[m,k] b[n,k] ),  per-tensor / per-row scales
//
// [FFS] "FP8 formats, scaling and LLM inference", section "Prefill 与 Decode 的收益不同"
// (Decode): with a small batch the linear layer is bound by reading the weight, and
// FP8 halves those bytes; the GEMM shape is too small to keep the tensor cores busy,
// and does not need to.  The kernel is built around streaming W once, at HBM speed,
// on every SM:
//   - W is the MMA's A operand (M = 128 weight rows per instruction) and the tokens
//     are its N (the token count rounded up to 16): D[n, m] = sum_k W X^T.  Each
//     instruction then consumes 4 KB of W, however few the tokens;
//   - W's rows are split into one contiguous range per CTA (one CTA per SM) in units
//     of 16 rows, as evenly as the units allow, and each range is done in chunks of
//     at most 128 rows.  Rows of the 128-row tile past a chunk are not loaded; their
//     accumulator lanes are never read.  No partial sums cross CTAs;
//   - HBM is read in long runs: a stage holds KBS (4, or 3 with more tokens) K blocks
//     of 128 bytes of the chunk, loaded as 64-row (and 16-row) TMA boxes issued
//     row-group by row-group, so each row's KBS consecutive blocks are requested back
//     to back.  (Measured on this part with loads alone: 128-row x 128-byte boxes
//     stream at ~4.8 TB/s, 64 rows x 4 consecutive blocks at ~6.2 TB/s.)  The boxes
//     land so that every K block is one K-major 128-byte-swizzled 128-row tile;
//   - X comes as one box per K block of the rounded-up token count (rows past M are
//     zero-filled by TMA); FP32 accumulators are double-buffered in TMEM across
//     chunks;
//   - the two epilogue warps of each TMEM lane quarter hold its 32 weight rows and
//     split the tokens in groups of 16: for each of its tokens a warp writes 32
//     consecutive outputs of Y's row (a 64-byte store per warp).
// Hopper-era decode kernels split K across CTAs (and reduce the partial sums) to
// occupy the machine; with per-SM ranges of whole rows W is read exactly once.
// Every wait is bounded as in the tiled kernels.
#include "gemm_common.cuh"

namespace fp8b {

constexpr int D_UNIT = 16;                 // rows of W per work unit
constexpr int D_TILE = 128;                // rows of W per MMA (the instruction's M)
constexpr int D_MAX_KBS = 4;
constexpr int D_MAX_STAGES = 8;
constexpr uint32_t D_TILE_BYTES = D_TILE * BK;          // 16 KB: one K block of a chunk
constexpr uint32_t D_BAR_BYTES = 1024;                  // barriers + misc, ahead of the stages
constexpr uint32_t D_SMEM = 227 * 1024;                 // dynamic shared memory budget

struct DecodeParams {
    int32_t units;         // ceil(N / 16)
    int32_t nt;            // tokens per MMA: M rounded up to 16
    int32_t kbs;           // K blocks per stage
    int32_t stages;
    uint32_t stage_bytes;  // kbs * (D_TILE_BYTES + nt * BK)
};

// The W rows of CTA c: units [u0, u0 + cnt) of 16 rows, done in chunks of <= 8 units.
struct DecodeRange {
    int32_t u0, cnt, nch;
};

__device__ __forceinline__ DecodeRange decode_range(int32_t units, int32_t c, int32_t ctas) {
    const int32_t base = units / ctas, extra = units % ctas;
    DecodeRange r;
    r.u0 = c * base + min(c, extra);
    r.cnt = base + (c < extra ? 1 : 0);
    r.nch = (r.cnt + 7) / 8;
    return r;
}

// Chunk j of a range: first row n0 and its row count w (a multiple of 16, <= 128).
__device__ __forceinline__ void decode_chunk(const DecodeRange& r, int32_t j, int32_t& n0, int32_t& w) {
    const int32_t ua = r.u0 + 8 * j;
    const int32_t ub = min(ua + 8, r.u0 + r.cnt);
    n0 = ua * D_UNIT;
    w = (ub - ua) * D_UNIT;
}

constexpr int D_EPI_WARPS = 8;             // two per TMEM lane quarter, each half of the tokens
constexpr int D_THREADS = 32 * (2 + D_EPI_WARPS);

template <bool EXT>
__global__ void __launch_bounds__(D_THREADS, 1)
fp8_decode_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW64,
                  const __grid_constant__ CUtensorMap tmW16, const GemmParams p, const DecodeParams d) {
    constexpr int EPI_WARPS = D_EPI_WARPS;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + D_MAX_STAGES;
    uint64_t* tfull = empty + D_MAX_STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* teardown = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(teardown + 1);
    volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);
    // stage s: KBS W tiles (16 KB each) at s * stage_bytes, then KBS X tiles (nt * 128 B each)
    uint8_t* stages = smem + D_BAR_BYTES;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const DecodeRange range = decode_range(d.units, blockIdx.x, gridDim.x);
    const int32_t S = d.stages;
    const int32_t nkc = (p.num_kb + d.kbs - 1) / d.kbs;       // stages per chunk
    const uint32_t x_off = (uint32_t)d.kbs * D_TILE_BYTES;    // X tiles within a stage

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], EPI_WARPS);
        }
        ptx::mbar_init(teardown, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmX);
        ptx::prefetch_tmap(&tmW64);
        ptx::prefetch_tmap(&tmW16);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, 256);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        // Step i of this CTA is K stage i % nkc of chunk i / nkc.  When the kernel runs
        // as the programmatic dependent of the kernel that quantised X (p.pdl), W cannot
        // be that kernel's output: the first ring of W loads goes out at once, and only
        // the X loads wait for the quantiser's results (pdl_wait).
        if (lane == 0) {
            const int32_t total = range.nch * nkc;
            const int32_t pre = p.pdl ? min(S, total) : 0;
            auto issue = [&](int32_t i, uint32_t stage, bool w_part, bool x_part) {
                int32_t n0, w;
                decode_chunk(range, i / nkc, n0, w);
                const int32_t kb0 = (i % nkc) * d.kbs;
                const int32_t kbs = min(d.kbs, p.num_kb - kb0);
                uint8_t* st = stages + stage * d.stage_bytes;
                if (w_part) {
                    ptx::mbar_arrive_expect_tx(&full[stage], (uint32_t)kbs * (uint32_t)(w + d.nt) * BK);
                    // row group by row group, each group's K blocks back to back
                    for (int32_t r = 0; r < w;) {
                        const bool big = w - r >= 64;
                        for (int32_t b = 0; b < kbs; ++b)
                            ptx::tma_load_2d(st + b * D_TILE_BYTES + r * BK, big ? &tmW64 : &tmW16, &full[stage],
                                             (kb0 + b) * BK, n0 + r);
                        r += big ? 64 : D_UNIT;
                    }
                }
                if (x_part)
                    for (int32_t b = 0; b < kbs; ++b)
                        ptx::tma_load_2d(st + x_off + b * d.nt * BK, &tmX, &full[stage], (kb0 + b) * BK, 0);
            };
            IssuedLoads loads;
            for (int32_t i = 0; i < pre; ++i) issue(i, (uint32_t)i, true, false);   // fresh ring: no waits
            pdl_wait();
            for (int32_t i = 0; i < pre; ++i) {
                issue(i, (uint32_t)i, false, true);
                loads.note((uint32_t)i, 0u);
            }
            uint32_t stage = (uint32_t)(pre % S), phase = (pre == S) ? 1u : 0u;
            for (int32_t i = pre; i < total; ++i) {
                if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.status, p.wait_ns)) break;
                issue(i, stage, true, true);
                loads.note(stage, phase);
                if (++stage == (uint32_t)S) { stage = 0; phase ^= 1u; }
            }
            loads.drain(full, p.status);      // loads in flight after an abort
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer: D[n, m] += W X^T
        uint32_t stage = 0, phase = 0, acc_it = 0;
        bool ok = true;
        const uint32_t s0 = ptx::smem_u32(stages);
        for (int32_t j = 0; j < range.nch && ok; ++j) {
            const uint32_t buf = acc_it & 1u, use = acc_it >> 1;
            if (!wait_bounded(&tempty[buf], (use & 1u) ^ 1u, abort_flag, p.status, p.wait_ns)) { ok = false; break; }
            ptx::tc_fence_after();
            for (int32_t kc = 0; kc < nkc; ++kc) {
                const int32_t kbs = min(d.kbs, p.num_kb - kc * d.kbs);
                if (!wait_bounded(&full[stage], phase, abort_flag, p.status, p.wait_ns)) { ok = false; break; }
                ptx::tc_fence_after();
                if (lane == 0) {
                    const uint32_t st = s0 + stage * d.stage_bytes;
                    for (int32_t b = 0; b < kbs; ++b) {
#pragma unroll
                        for (int k = 0; k < BK / UMMA_K; ++k) {
                            const uint64_t ad = ptx::sdesc_kmajor_sw128(st + b * D_TILE_BYTES + k * UMMA_K);
                            const uint64_t bd = ptx::sdesc_kmajor_sw128(st + x_off + b * d.nt * BK + k * UMMA_K);
                            ptx::mma_f8f6f4(tmem_base + buf * 128, ad, bd, p.idesc, (kc | b | k) != 0);
                        }
                    }
                    ptx::mma_commit(&empty[stage]);
                }
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
    } else {
        // ------------------------------------------------ epilogue: lane = weight row
        // two warps per TMEM lane quarter: warp half th takes the 16-token groups th, th + 2, ...
        pdl_wait();                           // X's scales (and epilogue inputs) may be just written
        const int quarter = warp & 3;
        const int th = (warp - 2) >> 2;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        uint32_t amax_bits = 0;               // |y| as fp32 patterns (order-preserving for y >= 0)
        float ys = 0.0f;
        bool yq_ok = false;
        if (EXT && p.yq) {
            ys = __ldg(p.yq_scale);
            yq_ok = ys >= 1.17549435e-38f && ys <= 8.5070592e37f;
            if (!yq_ok && lane == 0) report_status(p.status, FP8_ERR_INVALID_ARG);
        }
        uint32_t acc_it = 0;
        for (int32_t j = 0; j < range.nch; ++j) {
            int32_t n0, w;
            decode_chunk(range, j, n0, w);
            const uint32_t buf = acc_it & 1u, use = acc_it >> 1;
            if (!wait_bounded(&tfull[buf], use & 1u, abort_flag, p.status, p.wait_ns)) break;
            ptx::tc_fence_after();
            const int32_t r = quarter * 32 + lane;                 // row of the chunk
            const int32_t n = n0 + r;
            const bool valid = r < w && n < p.N;
            if (quarter * 32 < w) {                                // warp-uniform
                const float sw = valid ? __ldg(p.sb + (int64_t)n * p.sb_stride) : 0.0f;
                float bias = 0.0f;
                if (EXT && p.bias && valid) bias = bf16bits_to_float(__ldg(p.bias + n));
                for (int32_t c0 = 16 * th; c0 < p.M; c0 += 32) {
                    uint32_t acc[16];
                    ptx::tmem_ld_32x32b_x16(tmem_base + lane_base + buf * 128 + c0, acc);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        const int32_t m = c0 + t;
                        if (m >= p.M || !valid) continue;
                        float v = __uint_as_float(acc[t]) * (__ldg(p.sa + (int64_t)m * p.sa_stride) * sw);
                        if (EXT) v = __fadd_rn(v, bias);
                        const uint32_t yb = pack_bf16x2(v, 0.0f) & 0xFFFFu;
                        if (!EXT || p.write_y) p.y[(int64_t)m * p.ldy + n] = (uint16_t)yb;
                        if (EXT) {
                            amax_bits = max(amax_bits, (yb & 0x7FFFu) << 16);
                            if (yq_ok) {
                                // y / s_y rounded once (IEEE); a quotient beyond F_max saturates
                                const float q = __fdiv_rn(bf16bits_to_float(yb), ys);
                                const uint32_t code = p.yq_fmt == FP8_E4M3 ? cvt_pair<FP8_E4M3>(q, 0.0f)
                                                                          : cvt_pair<FP8_E5M2>(q, 0.0f);
                                p.yq[(int64_t)m * p.ldq + n] = (uint8_t)(code & 0xFFu);
                            }
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
            ++acc_it;
        }
        if (EXT && p.amax) {                   // every lane reaches this point
            const uint32_t m = __reduce_max_sync(0xffffffffu, amax_bits);
            if (lane == 0 && m != 0) atomicMax(p.amax, m);
        }
    }

    // ------------------------------------------------ teardown
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem_base, 256);
}

template <bool EXT>
static cudaError_t launch_decode_t(const GemmArgs& g, GemmParams p, cudaStream_t st) {
    DecodeParams d{};
    d.nt = (int32_t)((g.M + 15) / 16 * 16);
    d.units = (int32_t)((g.N + D_UNIT - 1) / D_UNIT);
    // 4 K blocks per stage (3 stages) up to 16 tokens; with more tokens the X tiles grow
    // and 3 blocks (3 stages) beat both 4 blocks (2 stages) and 2 blocks (5 stages)
    d.kbs = d.nt <= 16 ? D_MAX_KBS : 3;
    d.stage_bytes = (uint32_t)d.kbs * (D_TILE_BYTES + (uint32_t)d.nt * BK);
    d.stages = (int32_t)std::min<uint32_t>(D_MAX_STAGES, (D_SMEM - 1024 - D_BAR_BYTES) / d.stage_bytes);
    CUtensorMap tx, t64, t16;
    if (!make_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a, (uint64_t)g.K, (uint64_t)g.M, (uint64_t)g.K, BK,
                     (uint32_t)d.nt, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&t64, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.b, (uint64_t)g.K, (uint64_t)g.N, (uint64_t)g.K, BK, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&t16, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.b, (uint64_t)g.K, (uint64_t)g.N, (uint64_t)g.K, BK, 16,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    static bool attr_done[kDeviceCacheSlots];   // the attribute is set per device
    const int ds = device_slot();
    if (ds < 0 || !attr_done[ds]) {
        cudaError_t e = cudaFuncSetAttribute(fp8_decode_kernel<EXT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)D_SMEM);
        if (e != cudaSuccess) return e;
        if (ds >= 0) attr_done[ds] = true;
    }
    // request only what the stages use, so that a small kernel running just before (the
    // X quantize, whose dependent this kernel may be) can share an SM with this one
    const uint32_t smem = 1024 + D_BAR_BYTES + (uint32_t)d.stages * d.stage_bytes;
    // swapped operands: the instruction's A is W (format fmt_b), its B is X (fmt_a);
    // M = 128 weight rows, N = nt tokens
    p.idesc = (1u << 4) | ((uint32_t)g.fmt_b << 7) | ((uint32_t)g.fmt_a << 10) | ((uint32_t)(d.nt >> 3) << 17) |
              ((uint32_t)(D_TILE >> 4) << 24);
    const int grid = std::max(1, std::min(d.units, num_sms()));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(D_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.pdl ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, fp8_decode_kernel<EXT>, tx, t64, t16, p, d);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// M <= D_MAX_TOKENS, per-tensor / per-row scales (p holds the scales, epilogue
// options, output and K-block count).
cudaError_t launch_decode(const GemmArgs& g, const GemmParams& p, cudaStream_t st) {
    return p.ext ? launch_decode_t<true>(g, p, st) : launch_decode_t<false>(g, p, st);
}

}  // namespace fp8b
