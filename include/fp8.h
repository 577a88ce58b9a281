/*
 * fp8.h -- C ABI of libfp8.so, the B200 (sm_100a) FP8 runtime linear path.
 *
 * The path, as the source pages describe it:
 *   X --amax reduce--> a_max --scale--> s = a_max / F_max --clip and cast--> X_fp8
 *   Y = s_x * s_w * (X_fp8 W_fp8^T), FP32 accumulation, BF16 output.
 * Pages cited below:
 *   [FFS] "FP8 formats, scaling and LLM inference" (charlestar.github.io)
 *   [PQG] "FP8 产线量化落地指南" (m.xxqk.cn)
 *   [FPI] "FP8 推理：8 位浮点量化、E4M3/E5M2 与 NVIDIA FP8 生态" (plumephp.com)
 *   [FRLP] "41. FP8 Runtime Low Precision Paths" (datawhalechina llm-algo-leetcode)
 *
 * Conventions for every entry point
 *  - Pointers named *_dev are DEVICE pointers owned by the caller; the library
 *    allocates no device memory on these paths.  `stream` is a cudaStream_t
 *    (NULL = legacy default stream).  Work is enqueued asynchronously; nothing
 *    synchronises the host.
 *  - The returned status reports only the synchronous argument checks and launch
 *    errors.  Conditions found on the device are written to `dev_status` (a
 *    device int32 the caller zeroes; nullable): the first error code found is
 *    stored there, and the caller reads it after synchronising.
 *  - Layouts are row-major, last index contiguous.  X is [M, K] with row stride
 *    ld (elements); W is [N, K] (out x in, as nn.Linear stores it); Y = X W^T is
 *    [M, N] with row stride ldy.
 *  - Codes are 8-bit E4M3 ("fn": no Inf, NaN = S.1111.111) or E5M2 (IEEE-style
 *    Inf/NaN) with biases 7 / 15 and maxima 448 / 57344 ([FFS] section
 *    "8 个 Bit 怎样分配"; [FPI] section "数值特性").
 *  - Rounding is IEEE round-to-nearest-even everywhere; x/s is an fp32 IEEE
 *    division; values are clipped to +-F_max before the cast ([PQG] code step 3).
 *  - Inputs must be finite; a NaN/Inf input sets FP8_ERR_NONFINITE in dev_status
 *    and leaves the outputs unspecified ([FFS] section "数值验证看什么", non-finite).
 */
#ifndef FP8_B200_H
#define FP8_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FP8_ABI_VERSION 2

#if defined(__GNUC__)
#define FP8_API __attribute__((visibility("default")))
#else
#define FP8_API
#endif

typedef enum { FP8_E4M3 = 0, FP8_E5M2 = 1 } fp8_format_t;

/*
 * Scaling granularity ([FFS] sections "Per-tensor Scaling 的优点与问题",
 * "Per-channel 与 Block Scaling", "Current Scaling", "Delayed Scaling").
 * Scale buffer layout produced by fp8_quantize for a [rows, cols] input:
 *   TENSOR         float[1]
 *   ROW            float[rows]                 (per token for X, per output channel for W)
 *   BLOCK_1x128    float[rows][ceil(cols/128)]  (1 x 128 blocks along the row)
 *   BLOCK_128x128  float[ceil(rows/128)][ceil(cols/128)]
 *   MX32           uint8[rows][cols/32], E8M0 (2^(byte-127)), E4M3 codes only
 *   DELAYED        float[1], from the amax history (see fp8_history_t)
 * Every float scale is the dequantisation multiplier s = fp32(max(amax, 1e-12f) / F_max)
 * ([FFS] eq. s = a_max / F_max; [PQG] code: amax floor 1e-12); MX32 stores
 * e = clamp(floor(log2 amax) - 8, -127, 127) as the byte e + 127 (amax = 0 -> 0).
 */
typedef enum {
    FP8_SCALE_TENSOR = 0,
    FP8_SCALE_ROW = 1,
    FP8_SCALE_BLOCK_1x128 = 2,
    FP8_SCALE_BLOCK_128x128 = 3,
    FP8_SCALE_MX32 = 4,
    FP8_SCALE_DELAYED = 5
} fp8_scaling_t;

typedef enum {
    FP8_OK = 0,
    FP8_ERR_INVALID_ARG = 1,        /* a size, mode, format or pointer is invalid */
    FP8_ERR_ALIGNMENT = 2,          /* a pointer or stride breaks the 16-byte rules */
    FP8_ERR_UNSUPPORTED_DEVICE = 3, /* the current device is not compute capability 10.x */
    FP8_ERR_NONFINITE = 4,          /* (dev_status) a NaN/Inf input element was seen */
    FP8_ERR_TIMEOUT = 5,            /* (dev_status) a bounded device-side wait gave up */
    FP8_ERR_CUDA = 6,               /* a CUDA runtime/driver call failed */
    FP8_ERR_WORKSPACE = 7           /* workspace missing or smaller than fp8_workspace_size() */
} fp8_status_t;

/*
 * Amax history for delayed scaling ([FFS] section "Delayed Scaling":
 * s_{t+1} = f(a_t, ..., a_{t-h+1}) / F_max, with f = window maximum).
 *   ring_dev     float[len] on the device, zero before step 0.
 *   len          window length h (>= 1).
 *   step         host-side step counter t; fp8_quantize reads it and adds 1 after
 *                enqueueing the step.
 *   pending_dev  one device float, zero before step 0 (running amax of the step).
 *   ticket_dev   one device uint32, zero before step 0 (CTA arrival counter).
 * Step 0 has no history and uses current per-tensor scaling; step t >= 1 uses
 * s_t = max(max(ring), 1e-12f) / F_max.  After the step, ring[t mod h] holds the
 * raw amax of X_t, and pending/ticket are back to zero.  A step whose input holds a
 * NaN/Inf (FP8_ERR_NONFINITE in dev_status; that step's outputs are unspecified)
 * records nothing: ring[t mod h] keeps its previous value, so the bad step does
 * not set the scale of the h steps after it, and step still advances.  Two steps
 * on the same history must be stream-ordered.
 */
typedef struct {
    float* ring_dev;
    int32_t len;
    int64_t step;
    float* pending_dev;
    uint32_t* ticket_dev;
} fp8_history_t;

/* ABI version (FP8_ABI_VERSION). */
FP8_API int32_t fp8_abi_version(void);

/* Human-readable name of a status code (static storage). */
FP8_API const char* fp8_status_string(int32_t status);

/* FP8_OK when the current CUDA device is compute capability 10.x (sm_100a),
 * FP8_ERR_UNSUPPORTED_DEVICE otherwise, FP8_ERR_CUDA when CUDA is unusable.
 * (The device gate of [FRLP] section "5.2" preflight, moved to the library.)  Every
 * entry point that launches work applies the same gate first.  For tests, the
 * environment variable FP8_B200_FORCE_CC_MAJOR (a decimal number, read once per
 * process) replaces the device's compute capability major in the gate. */
FP8_API int32_t fp8_device_check(void);

/*
 * Workspace bytes an entry point needs.  which: 0 = fp8_quantize,
 * 1 = fp8_scaled_gemm, 2 = fp8_linear_forward.  For 0, (M, K) is the input
 * shape [rows, cols] and N is ignored.  The workspace needs no initialisation.
 * For per-tensor current scaling of a large dense tensor (>= 16 Mi elements) the
 * quantize runs as one cooperative launch whose CTAs exchange their amax through
 * the workspace; the workspace then keeps a call counter from one call to the next
 * (nothing else), so calls that share one workspace must not overlap on the GPU,
 * and after a call that reported FP8_ERR_TIMEOUT its contents are undefined until
 * the caller zeroes it.
 */
FP8_API size_t fp8_workspace_size(int32_t which, int64_t M, int64_t N, int64_t K, int32_t mode);

/*
 * fp8_quantize -- amax reduce + scale + clip + RNE cast (+ optional dequant).
 * [FFS] section "Scale 怎样把 Tensor 塞进 E4M3": X_fp8 = cast(clip(X / s)),
 * a_max = max|X|, s = a_max / F_max, X^ = s X_fp8; [PQG] section
 * "运行时动态张量缩放" and its code fp8_dynamic_quantize_tensor.
 *   x_dev        bf16 [rows, cols], row stride ld elements.  16-byte aligned, ld % 8 == 0.
 *   rows, cols   >= 0; cols % 16 == 0 (cols % 32 == 0 for MX32).  rows == 0 or
 *                cols == 0 still writes the scales (amax = 0 -> floor scale).
 *   fmt          FP8_E4M3 or FP8_E5M2 (MX32: E4M3 only).
 *   mode         fp8_scaling_t; DELAYED needs hist.
 *   q_dev        uint8 codes [rows, cols], dense (row stride cols), 16-byte aligned.
 *   scale_dev    scale buffer in the layout listed with fp8_scaling_t.
 *   hist         host struct, DELAYED only (else NULL); its step is advanced.
 *   dequant_dev  nullable; bf16 [rows, cols] dense, bf16_RNE(fp32(decode(q) * s)).
 *   dev_status   nullable device int32 (FP8_ERR_NONFINITE; FP8_ERR_TIMEOUT if the
 *                grid-wide amax exchange of the single-launch per-tensor kernel gave up).
 *   workspace_dev, ws_bytes  at least fp8_workspace_size(0, rows, 0, cols, mode) bytes
 *                (0 for modes other than TENSOR/DELAYED); 8-byte aligned for the
 *                single-launch per-tensor kernel (otherwise two passes run instead).
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED_DEVICE, WORKSPACE, CUDA.
 */
FP8_API int32_t fp8_quantize(const void* x_dev, int64_t rows, int64_t cols, int64_t ld,
                     int32_t fmt, int32_t mode, uint8_t* q_dev, void* scale_dev,
                     fp8_history_t* hist, void* dequant_dev, int32_t* dev_status,
                     void* workspace_dev, size_t ws_bytes, void* stream);

/*
 * fp8_scaled_gemm -- Y = bf16( sum_k S_a(m,k) a[m,k] * S_b(n,k) b[n,k] ) with FP32
 * accumulation on the tcgen05 tensor cores ([FFS] section
 * "一次 FP8 GEMM 的完整精度契约": Y ~= s_x s_w (X_8 W_8), wider accumulation,
 * BF16 output; [PQG] code fp8_gemm_forward, out_dtype bf16).
 *   a_dev [M, K] and b_dev [N, K]: codes, dense row-major (K contiguous), 16-byte aligned.
 *   a_scale_dev / b_scale_dev in the fp8_quantize layout for a_mode / b_mode.
 *   Mode pairs: a, b in {TENSOR, ROW, DELAYED} (DELAYED reads as TENSOR), any
 *   mix; (BLOCK_1x128, BLOCK_128x128); (MX32, MX32).
 *   fmt_a, fmt_b: E4M3 or E5M2 for the tensor/row modes; E4M3 for block and MX32.
 *   K % 16 == 0 (K % 32 == 0 for MX32); M, N >= 0; K == 0 writes zeros.
 *   y_dev bf16 [M, N], row stride ldy >= N.  With ldy % 8 == 0 and a 16-byte aligned
 *   y_dev the tiles leave through TMA stores; otherwise through plain stores.
 *   dev_status: nullable device int32; FP8_ERR_TIMEOUT if a pipeline wait gave up.
 * The workspace is unused (pass NULL, 0).
 */
FP8_API int32_t fp8_scaled_gemm(const uint8_t* a_dev, const void* a_scale_dev, int32_t a_mode, int32_t fmt_a,
                        const uint8_t* b_dev, const void* b_scale_dev, int32_t b_mode, int32_t fmt_b,
                        int64_t M, int64_t N, int64_t K, void* y_dev, int64_t ldy,
                        int32_t* dev_status, void* workspace_dev, size_t ws_bytes, void* stream);

/*
 * fp8_linear_forward -- one FP8 linear layer: quantize X with x_mode (current
 * scaling, or DELAYED with hist) into the workspace, then fp8_scaled_gemm with
 * the pre-quantised static weight ([PQG] section "运行时动态张量缩放": S_w fixed
 * offline, S_x computed per batch on the GPU; [FFS] section "Weight Scale 与
 * Activation Scale 生命周期不同").
 *   x_dev bf16 [M, K], row stride ldx.  x_mode: TENSOR, ROW, BLOCK_1x128, MX32
 *   or DELAYED; w_mode must pair with it as in fp8_scaled_gemm.
 *   w_dev/w_scale_dev: codes [N, K] and scales as fp8_quantize produced them.
 *   workspace: fp8_workspace_size(2, M, N, K, x_mode) bytes, 256-byte aligned.
 */
FP8_API int32_t fp8_linear_forward(const void* x_dev, int64_t M, int64_t K, int64_t ldx, int32_t x_fmt,
                           int32_t x_mode, fp8_history_t* hist,
                           const uint8_t* w_dev, const void* w_scale_dev, int32_t w_mode,
                           int32_t w_fmt, int64_t N, void* y_dev, int64_t ldy,
                           int32_t* dev_status, void* workspace_dev, size_t ws_bytes, void* stream);

/*
 * fp8_amax -- a_max = max |x| over a bf16 tensor, written as one fp32 to amax_dev
 * ([FFS] section "Scale 怎样把 Tensor 塞进 E4M3": a_max = max|X|).  Exact: the
 * largest bf16 magnitude is itself representable in fp32, and a maximum does not
 * depend on the reduction order.
 *   x_dev, rows, cols, ld  as for fp8_quantize (cols % 16 == 0, ld % 8 == 0,
 *                16-byte aligned); an empty tensor gives 0.
 *   amax_dev     device float, overwritten (needs no initialisation).
 *   dev_status   nullable; FP8_ERR_NONFINITE for a NaN/Inf element (amax_dev is
 *                then unspecified).
 *   workspace_dev, ws_bytes  fp8_workspace_size(0, rows, 0, cols, FP8_SCALE_TENSOR).
 * Together with fp8_quantize_with_amax this splits per-tensor current scaling at
 * its one global step, the amax reduction, so that a caller can combine maxima
 * from several places before the cast: shards of one tensor on several GPUs
 * (an all-reduce with MAX makes every shard use the scale of the whole tensor,
 * [FFS] section "Current Scaling": ranks synchronise so that all shards share
 * one scale), or the amax that a GEMM epilogue already produced (fp8_epilogue_t).
 */
FP8_API int32_t fp8_amax(const void* x_dev, int64_t rows, int64_t cols, int64_t ld, float* amax_dev,
                         int32_t* dev_status, void* workspace_dev, size_t ws_bytes, void* stream);

/*
 * fp8_quantize_with_amax -- the cast phase of per-tensor current scaling with a
 * given a_max: s = fp32(max(*amax_dev, 1e-12f) / F_max), q = RNE(clip(x / s,
 * +-F_max)), scale_dev[0] = s ([FFS] section "Scale 怎样把 Tensor 塞进 E4M3").
 * With *amax_dev = max|x| the codes, scale and dequant equal those of
 * fp8_quantize(..., FP8_SCALE_TENSOR, ...) bit for bit; a smaller a_max
 * saturates the elements beyond it to +-F_max.
 *   amax_dev     device float >= 0 read on the device (a NaN/Inf value sets
 *                FP8_ERR_NONFINITE; the outputs are then unspecified).
 *   q_dev, scale_dev (float[1]), dequant_dev (nullable), dev_status: as fp8_quantize.
 *   No workspace.  Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED_DEVICE, CUDA.
 */
FP8_API int32_t fp8_quantize_with_amax(const void* x_dev, int64_t rows, int64_t cols, int64_t ld, int32_t fmt,
                                       const float* amax_dev, uint8_t* q_dev, float* scale_dev, void* dequant_dev,
                                       int32_t* dev_status, void* stream);

/*
 * Epilogue options of fp8_scaled_gemm_ex / fp8_linear_forward_ex ([FFS] section
 * "一次 FP8 GEMM 的完整精度契约": the output dtype, the output scale /
 * requantisation when the next operator consumes FP8, and the bias fusion are
 * part of the GEMM's contract; when the next layer runs in FP8 the epilogue can
 * apply the output scale itself instead of writing BF16 and launching a separate
 * cast.  [PQG] code fp8_gemm_forward takes an optional bias).  Per output element,
 * with v the fp32 scaled accumulator of fp8_scaled_gemm:
 *   v' = fp32(v + bias[n])                      (bias_dev != NULL; else v' = v)
 *   y  = bf16_RNE(v')                           stored to y_dev unless y_dev is NULL
 *   amax_dev <- max(amax_dev, |y|)              (amax_dev != NULL)
 *   yq = RNE(clip(fp32(y) / s_y, +-F_max))      (yq_dev != NULL; s_y = *yq_scale_dev)
 * so that yq, amax and y are exactly what "store Y in bf16, then reduce its amax /
 * cast it with scale s_y" would give.
 *   bias_dev      nullable bf16 [N], 16-byte aligned.
 *   amax_dev      nullable device float holding a value >= 0 before the call (e.g. 0);
 *                 the maximum |y| over the output is folded in with an atomic max.
 *   yq_dev        nullable uint8 [M, ldq] codes of format yq_fmt (E4M3 or E5M2).
 *   yq_scale_dev  device float s_y, the dequantisation multiplier of yq, required
 *                 with yq_dev; a value that is not a positive normal fp32 with a
 *                 finite reciprocal sets FP8_ERR_INVALID_ARG in dev_status (codes
 *                 then unspecified).
 *   ldq           row stride of yq in bytes, >= N.
 * A NULL fp8_epilogue_t pointer, or one with every pointer NULL, is plain
 * fp8_scaled_gemm.  With yq_dev set, y_dev may be NULL (FP8 output only).
 */
typedef struct {
    const void* bias_dev;
    float* amax_dev;
    uint8_t* yq_dev;
    const float* yq_scale_dev;
    int32_t yq_fmt;
    int64_t ldq;
} fp8_epilogue_t;

/* fp8_scaled_gemm with the epilogue options above (epi nullable). */
FP8_API int32_t fp8_scaled_gemm_ex(const uint8_t* a_dev, const void* a_scale_dev, int32_t a_mode, int32_t fmt_a,
                                   const uint8_t* b_dev, const void* b_scale_dev, int32_t b_mode, int32_t fmt_b,
                                   int64_t M, int64_t N, int64_t K, void* y_dev, int64_t ldy,
                                   const fp8_epilogue_t* epi, int32_t* dev_status, void* workspace_dev,
                                   size_t ws_bytes, void* stream);

/* fp8_linear_forward with the epilogue options above (epi nullable). */
FP8_API int32_t fp8_linear_forward_ex(const void* x_dev, int64_t M, int64_t K, int64_t ldx, int32_t x_fmt,
                                      int32_t x_mode, fp8_history_t* hist,
                                      const uint8_t* w_dev, const void* w_scale_dev, int32_t w_mode,
                                      int32_t w_fmt, int64_t N, void* y_dev, int64_t ldy,
                                      const fp8_epilogue_t* epi, int32_t* dev_status,
                                      void* workspace_dev, size_t ws_bytes, void* stream);

/*
 * fp8_weight_only_linear -- weight-only FP8 linear for a few tokens:
 *   y[m, n] = bf16( s_w[n] * sum_k x[m, k] * decode(w[n, k]) )
 * with X in BF16 and only the weight in FP8 ([FFS] section "Weight-only FP8 与 W8A8
 * FP8": the weight is stored in FP8, the activation stays BF16, the kernel reads
 * the FP8 weight and converts it; the gain is the weight's memory and bandwidth).
 * X is not quantised; the weight codes are decoded on chip (exactly) and the
 * products are accumulated in FP32.  Up to 3 tokens the contraction runs on the
 * CUDA cores (a matrix-vector product bound by the weight's bytes); above that the
 * codes are converted to BF16 and multiplied on the BF16 tensor-core path.
 *   x_dev        bf16 [M, K], row stride ldx (ldx % 8 == 0), 16-byte aligned.
 *   M            0 <= M <= FP8_WEIGHT_ONLY_MAX_TOKENS (the decode regime; larger
 *                batches belong on fp8_linear_forward); K % 16 == 0.
 *   w_dev, w_scale_dev, w_mode, w_fmt: codes [N, K] and the TENSOR / ROW (or
 *                DELAYED, read as TENSOR) scale fp8_quantize produced; E4M3 or E5M2.
 *   y_dev        bf16 [M, N], row stride ldy >= N.  K == 0 writes zeros.
 *   dev_status   nullable; FP8_ERR_TIMEOUT if a pipeline wait gave up.
 * No workspace.  Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED_DEVICE, CUDA.
 */
#define FP8_WEIGHT_ONLY_MAX_TOKENS 64
FP8_API int32_t fp8_weight_only_linear(const void* x_dev, int64_t M, int64_t K, int64_t ldx, const uint8_t* w_dev,
                                       const void* w_scale_dev, int32_t w_mode, int32_t w_fmt, int64_t N,
                                       void* y_dev, int64_t ldy, int32_t* dev_status, void* stream);

/*
 * fp8_linear_forward_noalloc -- fp8_linear_forward for callers that cannot
 * allocate device memory.  (The source pages have no counterpart: this is a
 * deployment convenience of this library, not part of the method.)
 *
 * Some callers have no way to obtain a workspace: code running inside a host
 * program that owns all device memory and passes its plug-ins only their input
 * and output buffers, or code that must not call cudaMalloc because it can
 * synchronise the whole device.  This entry point takes the same arguments as
 * fp8_linear_forward except the workspace; its scratch (quantised X, X scales,
 * per-tensor amax partials) is a fixed array of FP8_NOALLOC_SCRATCH_BYTES of
 * device memory inside libfp8.so, present on every GPU that loads the library
 * until the process exits.  The call itself allocates nothing.
 *   - Size limit: fp8_workspace_size(2, M, N, K, x_mode) must not exceed
 *     FP8_NOALLOC_SCRATCH_BYTES (e.g. M*K up to ~4.1 million codes); larger
 *     inputs return FP8_ERR_WORKSPACE and enqueue nothing.
 *   - The first call on each device looks up the scratch's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture begins.  The address is kept for the life of the
 *     process: a cudaDeviceReset (or anything else that unloads the library's
 *     device code) after the first call is not supported.
 *   - All calls share the one scratch array, which keeps the last call's
 *     contents (nothing in it needs to start at zero).  Calls whose work can
 *     overlap on the GPU -- different streams, or unordered host threads -- race
 *     on it: order them on one stream.
 * Other arguments, errors and results: as fp8_linear_forward.
 */
#define FP8_NOALLOC_SCRATCH_BYTES 4194304
FP8_API int32_t fp8_linear_forward_noalloc(const void* x_dev, int64_t M, int64_t K, int64_t ldx, int32_t x_fmt,
                                           int32_t x_mode, fp8_history_t* hist,
                                           const uint8_t* w_dev, const void* w_scale_dev, int32_t w_mode,
                                           int32_t w_fmt, int64_t N, void* y_dev, int64_t ldy,
                                           int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FP8_B200_H */
