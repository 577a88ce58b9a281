/*
 * fp8_oracle.c -- plain, slow, obviously-correct CPU oracle for the FP8 runtime
 * linear path.  TEST INFRASTRUCTURE ONLY: it is loaded by the test-suite, by the
 * smoke check and by the benchmark's CPU-baseline leg, never by the product
 * library.  It shares no code, header, table or constant generator with the
 * CUDA path under fp8_dynamic_scaled_b200/csrc.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (float arithmetic is IEEE binary32 round-to-nearest-even; no contraction).
 *
 * Sources (pages are cited by title and section):
 *  [FFS]  "FP8 formats, scaling and LLM inference" (charlestar.github.io, 2026-08-01):
 *         section "8 个 Bit 怎样分配" (E4M3 = 1+4+3 bits, E5M2 = 1+5+2, maxima 448 / 57344);
 *         section "Scale 怎样把 Tensor 塞进 E4M3" (X_fp8 = cast(clip(X/s)), X^ = s*X_fp8,
 *         a_max = max|X|, s = a_max/F_max);
 *         section "Per-channel 与 Block Scaling" (s_g = a_g/F_max per block g);
 *         section "Delayed Scaling" (s_{t+1} = f(a_t..a_{t-h+1})/F_max, window max);
 *         section "一次 FP8 GEMM 的完整精度契约" (Y ~= s_x s_w (X_8 W_8), wider accumulation).
 *  [PQG]  "FP8 产线量化落地指南" (m.xxqk.cn): section "运行时动态张量缩放" and its code
 *         (amax floor 1e-12, scale = amax/448, clamp to +-448, cast to float8_e4m3fn,
 *         BF16 GEMM output).
 *  [FPI]  "FP8 推理：8 位浮点量化、E4M3/E5M2 与 NVIDIA FP8 生态" (plumephp.com):
 *         section "数值特性" (bias 7 / 15; E5M2 full Inf/NaN, E4M3 limited);
 *         section "量化流程" (x / s, round to an FP8 value, store).
 *
 * Readings where the pages are silent:
 *  - rounding is IEEE round-to-nearest, ties to even mantissa;
 *  - E4M3 is the "fn" variant: no Inf, NaN only at S.1111.111, subnormals kept;
 *  - E5M2 follows IEEE-754 binary conventions (Inf at S.11111.00, NaN above);
 *  - the scale is the fp32 value max(amax, 1e-12f) / F_max, and x/s is an fp32
 *    IEEE division (not a multiplication by the reciprocal);
 *  - negative values that round to zero keep their sign (code 0x80);
 *  - MX32: e = clamp(floor(log2 amax) - 8, -127, 127), byte = e + 127, amax = 0 -> e = -127;
 *  - delayed: step 0 uses the current amax, later steps the max over the ring,
 *    and amax_t of the raw input is written to ring[t mod h] after use.
 *
 * Parity status: every function here is pinned (tests/test_oracle_pins.py and
 * tests/test_oracle_epilogue_pins.py: printed examples under tests/golden, closed
 * forms, exact integer arithmetic, brute force); none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_E4M3 = 0, ORC_E5M2 = 1 };
enum {
    ORC_TENSOR = 0,
    ORC_ROW = 1,
    ORC_BLOCK_1x128 = 2,
    ORC_BLOCK_128x128 = 3,
    ORC_MX32 = 4,
    ORC_DELAYED = 5
};

/* ------------------------------------------------------------------ */
/* Format parameters, written out from the bit layouts on the pages.   */
/* ------------------------------------------------------------------ */
typedef struct {
    int ebits;    /* exponent field width */
    int mbits;    /* mantissa field width */
    int bias;     /* exponent bias */
    int emin;     /* exponent of the smallest normal: 1 - bias */
} orc_fmt;

static orc_fmt fmt_of(int fmt) {
    orc_fmt f;
    if (fmt == ORC_E4M3) { f.ebits = 4; f.mbits = 3; f.bias = 7; }
    else                 { f.ebits = 5; f.mbits = 2; f.bias = 15; }
    f.emin = 1 - f.bias;
    return f;
}

/* Largest finite magnitude, derived from the field layout:
 * E4M3fn: the top exponent field is still finite except mantissa 111 (NaN),
 * so max = 1.110b * 2^(15-7) = 448.  E5M2: the top exponent field is Inf/NaN,
 * so max = 1.11b * 2^(30-15) = 57344. */
double orc_fmax(int fmt) {
    orc_fmt f = fmt_of(fmt);
    if (fmt == ORC_E4M3) {
        int emax = (1 << f.ebits) - 1 - f.bias;              /* 8 */
        double mant = 1.0 + (double)((1 << f.mbits) - 2) / (1 << f.mbits); /* 1.75 */
        return ldexp(mant, emax);
    } else {
        int emax = (1 << f.ebits) - 2 - f.bias;              /* 15 */
        double mant = 1.0 + (double)((1 << f.mbits) - 1) / (1 << f.mbits); /* 1.75 */
        return ldexp(mant, emax);
    }
}

/* ------------------------------------------------------------------ */
/* Decode: 8-bit code -> real value (double, exact).                  */
/* ------------------------------------------------------------------ */
double orc_decode(uint8_t code, int fmt) {
    orc_fmt f = fmt_of(fmt);
    int s = code >> 7;
    int e = (code >> f.mbits) & ((1 << f.ebits) - 1);
    int m = code & ((1 << f.mbits) - 1);
    double sign = s ? -1.0 : 1.0;
    int etop = (1 << f.ebits) - 1;
    if (fmt == ORC_E4M3) {
        if (e == etop && m == (1 << f.mbits) - 1) return NAN;
    } else {
        if (e == etop) return m == 0 ? sign * INFINITY : NAN;
    }
    if (e == 0) /* subnormal: m * 2^(emin - mbits) */
        return sign * ldexp((double)m, f.emin - f.mbits);
    return sign * ldexp(1.0 + (double)m / (1 << f.mbits), e - f.bias);
}

/* 1 when the code is a finite value (zero included). */
int orc_is_finite_code(uint8_t code, int fmt) {
    return isfinite(orc_decode(code, fmt)) ? 1 : 0;
}

/* ------------------------------------------------------------------ */
/* Encode, arithmetic form: finite v with |v| <= F_max -> nearest code */
/* under round-to-nearest-even.  Works in double, where every step is  */
/* exact for the float inputs the path produces.                        */
/* ------------------------------------------------------------------ */
uint8_t orc_encode(double v, int fmt) {
    orc_fmt f = fmt_of(fmt);
    int sign = signbit(v) ? 1 : 0;
    double a = fabs(v);
    int E;  /* exponent of the binade that holds a, or emin for subnormals */
    if (a < ldexp(1.0, f.emin)) {
        E = f.emin;
    } else {
        int ex;
        frexp(a, &ex);   /* a = fr * 2^ex, fr in [0.5, 1) -> floor(log2 a) = ex - 1 */
        E = ex - 1;
    }
    double quantum = ldexp(1.0, E - f.mbits);
    double n = a / quantum;          /* exact: division by a power of two */
    double r = rint(n);              /* default rounding mode: nearest, ties to even */
    double value = r * quantum;      /* exact */

    /* Re-derive the fields from the rounded value; this covers the carry into
     * the next binade (r == 2^(mbits+1)). */
    int e_field, m_field;
    if (value == 0.0) {
        e_field = 0; m_field = 0;
    } else if (value < ldexp(1.0, f.emin)) {
        e_field = 0;
        m_field = (int)(value / ldexp(1.0, f.emin - f.mbits));
    } else {
        int ex;
        frexp(value, &ex);
        int Ev = ex - 1;
        e_field = Ev + f.bias;
        m_field = (int)((value / ldexp(1.0, Ev) - 1.0) * (1 << f.mbits));
    }
    return (uint8_t)((sign << 7) | (e_field << f.mbits) | m_field);
}

/* ------------------------------------------------------------------ */
/* Encode, brute-force form: search all 256 codes of v's sign for the  */
/* nearest finite value; on an exact tie take the even code (mantissa  */
/* LSB 0).  Independent of orc_encode; the tests compare the two.      */
/* ------------------------------------------------------------------ */
uint8_t orc_encode_bruteforce(double v, int fmt) {
    int sign = signbit(v) ? 1 : 0;
    double a = fabs(v);
    int best = -1;
    double best_d = 0.0;
    for (int c = 0; c < 128; ++c) {
        uint8_t code = (uint8_t)((sign << 7) | c);
        double dv = orc_decode(code, fmt);
        if (!isfinite(dv)) continue;
        double d = fabs(fabs(dv) - a);
        if (best < 0 || d < best_d || (d == best_d && (code & 1) == 0)) {
            best = code;
            best_d = d;
        }
    }
    return (uint8_t)best;
}

/* ------------------------------------------------------------------ */
/* bf16 <-> fp32 and fp32 -> bf16 round-to-nearest-even.               */
/* ------------------------------------------------------------------ */
static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float x;
    memcpy(&x, &u, 4);
    return x;
}

uint16_t orc_f32_to_bf16(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    if (isnan(x)) return (uint16_t)((u >> 16) | 0x40);
    /* Keep the top 16 bits; round the dropped 16 bits to nearest, ties to the
     * even kept pattern. */
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xFFFFu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1;
    return (uint16_t)kept;
}

/* ------------------------------------------------------------------ */
/* Scale rules.                                                        */
/* ------------------------------------------------------------------ */
/* s = fp32(max(amax, 1e-12f) / F_max): [FFS] "Scale 怎样把 Tensor 塞进 E4M3" and
 * [PQG] code (clamp(amax, min=1e-12), scale = amax / FP8_E4M3_MAX). */
float orc_scale_from_amax(float amax, int fmt) {
    float floor_ = 1e-12f;
    float a = amax > floor_ ? amax : floor_;
    float F = (float)orc_fmax(fmt);
    return a / F;
}

/* MX32 shared exponent: e = clamp(floor(log2 amax) - 8, -127, 127); byte = e + 127. */
int orc_mx_exponent(float amax) {
    if (amax == 0.0f) return -127;
    int ex;
    frexp((double)amax, &ex);          /* exact floor(log2) for any positive float */
    int e = (ex - 1) - 8;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* Quantize one value with an fp32 scale: t = fp32(x / s), clip to +-F, encode. */
static uint8_t quant_one(float x, float s, int fmt, int* saturated) {
    float F = (float)orc_fmax(fmt);
    float t = x / s;
    if (saturated && fabsf(t) > F) *saturated += 1;
    float c = t;
    if (c > F) c = F;
    if (c < -F) c = -F;
    return orc_encode((double)c, fmt);
}

/* Quantize one value with a power-of-two scale 2^e: t = fp32(x * 2^-e) (the
 * product is exact in double and rounded once to fp32), clip, encode. */
static uint8_t quant_one_mx(float x, int e, int fmt) {
    float F = (float)orc_fmax(fmt);
    float t = (float)((double)x * ldexp(1.0, -e));
    float c = t;
    if (c > F) c = F;
    if (c < -F) c = -F;
    return orc_encode((double)c, fmt);
}

/* dequant = bf16_RNE(fp32(decode(q) * s)): [FFS] X^ = s X_fp8; [FPI] "反量化示例". */
static uint16_t dequant_one(uint8_t q, float s, int fmt) {
    float d = (float)orc_decode(q, fmt);
    float p = d * s;
    return orc_f32_to_bf16(p);
}

static int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

/* Number of scale entries the given mode produces for a [rows, cols] tensor. */
int64_t orc_scale_count(int mode, int64_t rows, int64_t cols) {
    switch (mode) {
    case ORC_TENSOR: case ORC_DELAYED: return 1;
    case ORC_ROW: return rows;
    case ORC_BLOCK_1x128: return rows * cdiv(cols, 128);
    case ORC_BLOCK_128x128: return cdiv(rows, 128) * cdiv(cols, 128);
    case ORC_MX32: return rows * (cols / 32);
    default: return -1;
    }
}

/* ------------------------------------------------------------------ */
/* amax over a rectangular region of a bf16 matrix.                    */
/* ------------------------------------------------------------------ */
static float amax_region(const uint16_t* x, int64_t ld, int64_t r0, int64_t r1,
                         int64_t c0, int64_t c1) {
    float m = 0.0f;
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t c = c0; c < c1; ++c) {
            float v = fabsf(bf16_to_f32(x[r * ld + c]));
            if (v > m) m = v;
        }
    return m;
}

/* Returns 0 on success, 1 on a non-finite input, 2 on a bad argument. */
static int check_finite(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            if (!isfinite(bf16_to_f32(x[r * ld + c]))) return 1;
    return 0;
}

/*
 * orc_quantize: the quantize step for every scaling mode except DELAYED
 * (see orc_delayed_step).
 *   x        bf16 [rows, cols] with row stride ld (elements)
 *   q        uint8 codes [rows, cols], dense
 *   scale    TENSOR: float[1]; ROW: float[rows]; BLOCK_1x128: float[rows][ceil(cols/128)];
 *            BLOCK_128x128: float[ceil(rows/128)][ceil(cols/128)]; MX32: uint8[rows][cols/32]
 *   dequant  optional bf16 [rows, cols] (NULL to skip)
 * Returns 0, 1 (non-finite input) or 2 (bad argument).
 */
int orc_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int fmt, int mode,
                 uint8_t* q, void* scale, uint16_t* dequant) {
    if (rows < 0 || cols < 0 || ld < cols) return 2;
    if (fmt != ORC_E4M3 && fmt != ORC_E5M2) return 2;
    if (mode == ORC_MX32 && (fmt != ORC_E4M3 || cols % 32 != 0)) return 2;
    if (check_finite(x, rows, cols, ld)) return 1;
    if (mode == ORC_TENSOR) {
        float a = amax_region(x, ld, 0, rows, 0, cols);
        float s = orc_scale_from_amax(a, fmt);
        ((float*)scale)[0] = s;
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t c = 0; c < cols; ++c) {
                uint8_t code = quant_one(bf16_to_f32(x[r * ld + c]), s, fmt, NULL);
                q[r * cols + c] = code;
                if (dequant) dequant[r * cols + c] = dequant_one(code, s, fmt);
            }
        return 0;
    }
    if (mode == ORC_ROW) {
        for (int64_t r = 0; r < rows; ++r) {
            float s = orc_scale_from_amax(amax_region(x, ld, r, r + 1, 0, cols), fmt);
            ((float*)scale)[r] = s;
            for (int64_t c = 0; c < cols; ++c) {
                uint8_t code = quant_one(bf16_to_f32(x[r * ld + c]), s, fmt, NULL);
                q[r * cols + c] = code;
                if (dequant) dequant[r * cols + c] = dequant_one(code, s, fmt);
            }
        }
        return 0;
    }
    if (mode == ORC_BLOCK_1x128 || mode == ORC_BLOCK_128x128) {
        int64_t bh = mode == ORC_BLOCK_1x128 ? 1 : 128;
        int64_t nbr = cdiv(rows, bh), nbc = cdiv(cols, 128);
        for (int64_t br = 0; br < nbr; ++br)
            for (int64_t bc = 0; bc < nbc; ++bc) {
                int64_t r0 = br * bh, r1 = r0 + bh < rows ? r0 + bh : rows;
                int64_t c0 = bc * 128, c1 = c0 + 128 < cols ? c0 + 128 : cols;
                float s = orc_scale_from_amax(amax_region(x, ld, r0, r1, c0, c1), fmt);
                ((float*)scale)[br * nbc + bc] = s;
                for (int64_t r = r0; r < r1; ++r)
                    for (int64_t c = c0; c < c1; ++c) {
                        uint8_t code = quant_one(bf16_to_f32(x[r * ld + c]), s, fmt, NULL);
                        q[r * cols + c] = code;
                        if (dequant) dequant[r * cols + c] = dequant_one(code, s, fmt);
                    }
            }
        return 0;
    }
    if (mode == ORC_MX32) {
        int64_t ng = cols / 32;
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t g = 0; g < ng; ++g) {
                int e = orc_mx_exponent(amax_region(x, ld, r, r + 1, g * 32, g * 32 + 32));
                ((uint8_t*)scale)[r * ng + g] = (uint8_t)(e + 127);
                float s2 = (float)ldexp(1.0, e);
                for (int64_t c = g * 32; c < g * 32 + 32; ++c) {
                    uint8_t code = quant_one_mx(bf16_to_f32(x[r * ld + c]), e, fmt);
                    q[r * cols + c] = code;
                    if (dequant) dequant[r * cols + c] = dequant_one(code, s2, fmt);
                }
            }
        return 0;
    }
    return 2;
}

/*
 * orc_delayed_step: one step t of delayed per-tensor scaling ([FFS] "Delayed Scaling").
 *   ring[len] holds the amax history (zero-initialised by the caller).
 *   t == 0: no history yet -> the scale comes from the current amax.
 *   t >= 1: s_t = max(max(ring), 1e-12f) / F_max.
 *   After quantizing, ring[t mod len] <- amax_t (raw amax of this step's input).
 *   *saturated receives the number of elements with |x / s_t| > F_max.
 *   *scale_out receives s_t.
 */
int orc_delayed_step(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int fmt,
                     float* ring, int32_t len, int64_t t, uint8_t* q, float* scale_out,
                     uint16_t* dequant, int64_t* saturated) {
    if (rows < 0 || cols < 0 || ld < cols || len <= 0 || t < 0) return 2;
    if (fmt != ORC_E4M3 && fmt != ORC_E5M2) return 2;
    if (check_finite(x, rows, cols, ld)) return 1;
    float amax_t = amax_region(x, ld, 0, rows, 0, cols);
    float s;
    if (t == 0) {
        s = orc_scale_from_amax(amax_t, fmt);
    } else {
        float h = 0.0f;
        for (int32_t i = 0; i < len; ++i) if (ring[i] > h) h = ring[i];
        s = orc_scale_from_amax(h, fmt);
    }
    int sat = 0;
    int64_t sat_total = 0;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            sat = 0;
            uint8_t code = quant_one(bf16_to_f32(x[r * ld + c]), s, fmt, &sat);
            sat_total += sat;
            q[r * cols + c] = code;
            if (dequant) dequant[r * cols + c] = dequant_one(code, s, fmt);
        }
    *scale_out = s;
    if (saturated) *saturated = sat_total;
    ring[t % len] = amax_t;
    return 0;
}

/* ------------------------------------------------------------------ */
/* GEMM reference ([FFS] "一次 FP8 GEMM 的完整精度契约"):                  */
/*   y[m,n] = sum_k (S_a(m,k) a[m,k]) (S_b(n,k) b[n,k])  in double,     */
/*   bound[m,n] = sum_k |same product|.                                 */
/* a: codes [M,K], b: codes [N,K] (W in out x in layout), Y = A B^T.    */
/* ------------------------------------------------------------------ */
static double scale_at(const void* scale, int mode, int64_t r, int64_t k, int64_t K) {
    switch (mode) {
    case ORC_TENSOR: case ORC_DELAYED: return ((const float*)scale)[0];
    case ORC_ROW: return ((const float*)scale)[r];
    case ORC_BLOCK_1x128: return ((const float*)scale)[r * cdiv(K, 128) + k / 128];
    case ORC_BLOCK_128x128: return ((const float*)scale)[(r / 128) * cdiv(K, 128) + k / 128];
    case ORC_MX32: return ldexp(1.0, (int)((const uint8_t*)scale)[r * (K / 32) + k / 32] - 127);
    default: return NAN;
    }
}

/* Dequantised operand row: out[k] = S(r,k) * decode(code[r,k]). */
static void deq_row(const uint8_t* codes, const void* scale, int mode, int fmt, int64_t r,
                    int64_t K, double* out) {
    for (int64_t k = 0; k < K; ++k)
        out[k] = scale_at(scale, mode, r, k, K) * orc_decode(codes[r * K + k], fmt);
}

/* Reference at a list of output points (m[i], n[i]). */
int orc_gemm_ref_points(const uint8_t* a, const void* sa, int a_mode, int fmt_a,
                        const uint8_t* b, const void* sb, int b_mode, int fmt_b,
                        int64_t M, int64_t N, int64_t K,
                        const int64_t* pm, const int64_t* pn, int64_t npts,
                        double* y, double* bound) {
    double* ra = (double*)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
    double* rb = (double*)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
    if (!ra || !rb) { free(ra); free(rb); return 2; }
    int64_t cur_m = -1;
    for (int64_t i = 0; i < npts; ++i) {
        int64_t m = pm[i], n = pn[i];
        if (m < 0 || m >= M || n < 0 || n >= N) { free(ra); free(rb); return 2; }
        if (m != cur_m) { deq_row(a, sa, a_mode, fmt_a, m, K, ra); cur_m = m; }
        deq_row(b, sb, b_mode, fmt_b, n, K, rb);
        double acc = 0.0, bnd = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double p = ra[k] * rb[k];
            acc += p;
            bnd += fabs(p);
        }
        y[i] = acc;
        bound[i] = bnd;
    }
    free(ra);
    free(rb);
    return 0;
}

/* Full reference for small problems: y and bound are [M, N]. */
int orc_gemm_ref_full(const uint8_t* a, const void* sa, int a_mode, int fmt_a,
                      const uint8_t* b, const void* sb, int b_mode, int fmt_b,
                      int64_t M, int64_t N, int64_t K, double* y, double* bound) {
    double* da = (double*)malloc(sizeof(double) * (size_t)(M * K > 0 ? M * K : 1));
    double* db = (double*)malloc(sizeof(double) * (size_t)(N * K > 0 ? N * K : 1));
    if (!da || !db) { free(da); free(db); return 2; }
    for (int64_t m = 0; m < M; ++m) deq_row(a, sa, a_mode, fmt_a, m, K, da + m * K);
    for (int64_t n = 0; n < N; ++n) deq_row(b, sb, b_mode, fmt_b, n, K, db + n * K);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, bnd = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = da[m * K + k] * db[n * K + k];
                acc += p;
                bnd += fabs(p);
            }
            y[m * N + n] = acc;
            bound[m * N + n] = bnd;
        }
    free(da);
    free(db);
    return 0;
}

/* Decoded values of every code of a format, for table-driven checks. */
void orc_decode_table(int fmt, double* out256) {
    for (int c = 0; c < 256; ++c) out256[c] = orc_decode((uint8_t)c, fmt);
}

/* Vector helpers so the tests can drive large arrays through ctypes. */
void orc_encode_array(const float* v, int64_t n, int fmt, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_encode((double)v[i], fmt);
}
void orc_encode_bruteforce_array(const float* v, int64_t n, int fmt, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_encode_bruteforce((double)v[i], fmt);
}
void orc_f32_to_bf16_array(const float* v, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f32_to_bf16(v[i]);
}
/* Quantize an array of fp32 values with one fp32 scale: t = x/s, clip, encode. */
/* Dequantised bf16 of codes under one fp32 scale: bf16_RNE(fp32(decode(q) * s)). */
void orc_dequant_scaled_array(const uint8_t* q, int64_t n, float s, int fmt, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = dequant_one(q[i], s, fmt);
}
void orc_quant_scaled_array(const float* v, int64_t n, float s, int fmt, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = quant_one(v[i], s, fmt, NULL);
}
