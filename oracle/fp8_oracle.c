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
 *    and amax_t of the raw input is written to ring[t mod h] after use; a step
 *    whose input holds a NaN/Inf is refused and writes nothing to the ring.
 *  - threads: rows (row blocks, output points) may be split over threads; every
 *    element is computed by the same code, so the results do not depend on it.
 *
 * Parity status: every function here is pinned (tests/test_oracle_pins.py and
 * tests/test_oracle_epilogue_pins.py: printed examples under tests/golden, closed
 * forms, exact integer arithmetic, brute force); none is "parity unpinned".
 */
#include <math.h>
#include <pthread.h>
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
/* Threads.  The array-wide entry points split their rows (row blocks,  */
/* output points) into contiguous ranges, one per thread.  Every        */
/* element is still produced by the same code, and a maximum or a count */
/* does not depend on how the ranges are combined, so the results are   */
/* the same for every thread count.  Default: 1 thread.                 */
/* ------------------------------------------------------------------ */
#define ORC_MAX_THREADS 256
static int g_threads = 1;

void orc_set_threads(int n) { g_threads = n < 1 ? 1 : (n > ORC_MAX_THREADS ? ORC_MAX_THREADS : n); }
int orc_get_threads(void) { return g_threads; }

typedef void (*orc_range_fn)(void* ctx, int64_t i0, int64_t i1, int part);
typedef struct {
    orc_range_fn fn;
    void* ctx;
    int64_t i0, i1;
    int part;
} orc_job;

static void* orc_job_main(void* p) {
    orc_job* j = (orc_job*)p;
    j->fn(j->ctx, j->i0, j->i1, j->part);
    return NULL;
}

/* Run fn on [0, n) cut into at most g_threads ranges whose bounds are multiples of
 * `grain`; range k gets part index k.  Returns the number of ranges. */
static int orc_parallel(int64_t n, int64_t grain, void* ctx, orc_range_fn fn) {
    if (n <= 0) return 0;
    if (grain < 1) grain = 1;
    int64_t units = (n + grain - 1) / grain;
    int parts = g_threads;
    if (parts > units) parts = (int)units;
    if (parts <= 1) {
        fn(ctx, 0, n, 0);
        return 1;
    }
    orc_job jobs[ORC_MAX_THREADS];
    pthread_t th[ORC_MAX_THREADS];
    int started[ORC_MAX_THREADS];
    for (int k = 0; k < parts; ++k) {
        int64_t u0 = units * k / parts, u1 = units * (k + 1) / parts;
        jobs[k].fn = fn;
        jobs[k].ctx = ctx;
        jobs[k].i0 = u0 * grain;
        jobs[k].i1 = u1 * grain < n ? u1 * grain : n;
        jobs[k].part = k;
    }
    for (int k = 1; k < parts; ++k) started[k] = pthread_create(&th[k], NULL, orc_job_main, &jobs[k]) == 0;
    fn(ctx, jobs[0].i0, jobs[0].i1, 0);
    for (int k = 1; k < parts; ++k) {
        if (started[k]) pthread_join(th[k], NULL);
        else fn(ctx, jobs[k].i0, jobs[k].i1, k);   /* no thread: run the range here */
    }
    return parts;
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

/* State shared by the row-range workers of orc_quantize / orc_delayed_step. */
typedef struct {
    const uint16_t* x;
    int64_t rows, cols, ld;
    int fmt;
    uint8_t* q;
    void* scale;
    uint16_t* dequant;
    float s;                              /* per-tensor scale of the cast */
    float amax_part[ORC_MAX_THREADS];     /* per-range amax */
    int64_t sat_part[ORC_MAX_THREADS];    /* per-range count of |x / s| > F_max */
    int bad_part[ORC_MAX_THREADS];        /* per-range: a non-finite element seen */
} qjob;

static void finite_rows(void* c, int64_t r0, int64_t r1, int part) {
    qjob* j = (qjob*)c;
    int bad = 0;
    for (int64_t r = r0; r < r1 && !bad; ++r)
        for (int64_t k = 0; k < j->cols; ++k)
            if (!isfinite(bf16_to_f32(j->x[r * j->ld + k]))) { bad = 1; break; }
    j->bad_part[part] = bad;
}

/* 1 when any element of x is NaN or Inf. */
static int check_finite(qjob* j) {
    int parts = orc_parallel(j->rows, 1, j, finite_rows);
    for (int k = 0; k < parts; ++k)
        if (j->bad_part[k]) return 1;
    return 0;
}

static void amax_rows(void* c, int64_t r0, int64_t r1, int part) {
    qjob* j = (qjob*)c;
    j->amax_part[part] = amax_region(j->x, j->ld, r0, r1, 0, j->cols);
}

/* a_max over the whole tensor: the maximum of the ranges' maxima. */
static float amax_all(qjob* j) {
    int parts = orc_parallel(j->rows, 1, j, amax_rows);
    float m = 0.0f;
    for (int k = 0; k < parts; ++k)
        if (j->amax_part[k] > m) m = j->amax_part[k];
    return m;
}

/* Cast rows [r0, r1) with the one scale j->s, counting saturated elements. */
static void cast_rows(void* c, int64_t r0, int64_t r1, int part) {
    qjob* j = (qjob*)c;
    int64_t sat_total = 0;
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t k = 0; k < j->cols; ++k) {
            int sat = 0;
            uint8_t code = quant_one(bf16_to_f32(j->x[r * j->ld + k]), j->s, j->fmt, &sat);
            sat_total += sat;
            j->q[r * j->cols + k] = code;
            if (j->dequant) j->dequant[r * j->cols + k] = dequant_one(code, j->s, j->fmt);
        }
    j->sat_part[part] = sat_total;
}

/* ROW: one scale per row. */
static void row_rows(void* c, int64_t r0, int64_t r1, int part) {
    (void)part;
    qjob* j = (qjob*)c;
    for (int64_t r = r0; r < r1; ++r) {
        float s = orc_scale_from_amax(amax_region(j->x, j->ld, r, r + 1, 0, j->cols), j->fmt);
        ((float*)j->scale)[r] = s;
        for (int64_t k = 0; k < j->cols; ++k) {
            uint8_t code = quant_one(bf16_to_f32(j->x[r * j->ld + k]), s, j->fmt, NULL);
            j->q[r * j->cols + k] = code;
            if (j->dequant) j->dequant[r * j->cols + k] = dequant_one(code, s, j->fmt);
        }
    }
}

/* BLOCK_1x128 (bh = 1) and BLOCK_128x128 (bh = 128): one scale per bh x 128 block
 * (ragged blocks at the right and bottom edges); i0..i1 index block rows. */
static void block_rows(qjob* j, int64_t bh, int64_t br0, int64_t br1) {
    int64_t nbc = cdiv(j->cols, 128);
    for (int64_t br = br0; br < br1; ++br)
        for (int64_t bc = 0; bc < nbc; ++bc) {
            int64_t r0 = br * bh, r1 = r0 + bh < j->rows ? r0 + bh : j->rows;
            int64_t c0 = bc * 128, c1 = c0 + 128 < j->cols ? c0 + 128 : j->cols;
            float s = orc_scale_from_amax(amax_region(j->x, j->ld, r0, r1, c0, c1), j->fmt);
            ((float*)j->scale)[br * nbc + bc] = s;
            for (int64_t r = r0; r < r1; ++r)
                for (int64_t k = c0; k < c1; ++k) {
                    uint8_t code = quant_one(bf16_to_f32(j->x[r * j->ld + k]), s, j->fmt, NULL);
                    j->q[r * j->cols + k] = code;
                    if (j->dequant) j->dequant[r * j->cols + k] = dequant_one(code, s, j->fmt);
                }
        }
}
static void block1_rows(void* c, int64_t i0, int64_t i1, int part) { (void)part; block_rows((qjob*)c, 1, i0, i1); }
static void block128_rows(void* c, int64_t i0, int64_t i1, int part) { (void)part; block_rows((qjob*)c, 128, i0, i1); }

/* MX32: one power-of-two scale per 32 consecutive elements of a row. */
static void mx_rows(void* c, int64_t r0, int64_t r1, int part) {
    (void)part;
    qjob* j = (qjob*)c;
    int64_t ng = j->cols / 32;
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t g = 0; g < ng; ++g) {
            int e = orc_mx_exponent(amax_region(j->x, j->ld, r, r + 1, g * 32, g * 32 + 32));
            ((uint8_t*)j->scale)[r * ng + g] = (uint8_t)(e + 127);
            float s2 = (float)ldexp(1.0, e);
            for (int64_t k = g * 32; k < g * 32 + 32; ++k) {
                uint8_t code = quant_one_mx(bf16_to_f32(j->x[r * j->ld + k]), e, j->fmt);
                j->q[r * j->cols + k] = code;
                if (j->dequant) j->dequant[r * j->cols + k] = dequant_one(code, s2, j->fmt);
            }
        }
}

/*
 * orc_quantize: the quantize step for every scaling mode except DELAYED
 * (see orc_delayed_step).
 *   x        bf16 [rows, cols] with row stride ld (elements)
 *   q        uint8 codes [rows, cols], dense
 *   scale    TENSOR: float[1]; ROW: float[rows]; BLOCK_1x128: float[rows][ceil(cols/128)];
 *            BLOCK_128x128: float[ceil(rows/128)][ceil(cols/128)]; MX32: uint8[rows][cols/32]
 *   dequant  optional bf16 [rows, cols] (NULL to skip)
 * Returns 0, 1 (non-finite input; nothing is written) or 2 (bad argument).
 */
int orc_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int fmt, int mode,
                 uint8_t* q, void* scale, uint16_t* dequant) {
    if (rows < 0 || cols < 0 || ld < cols) return 2;
    if (fmt != ORC_E4M3 && fmt != ORC_E5M2) return 2;
    if (mode < ORC_TENSOR || mode > ORC_MX32) return 2;
    if (mode == ORC_MX32 && (fmt != ORC_E4M3 || cols % 32 != 0)) return 2;
    qjob* j = (qjob*)calloc(1, sizeof(qjob));
    if (!j) return 2;
    j->x = x; j->rows = rows; j->cols = cols; j->ld = ld; j->fmt = fmt;
    j->q = q; j->scale = scale; j->dequant = dequant;
    int rc = 0;
    if (check_finite(j)) {
        rc = 1;
    } else if (mode == ORC_TENSOR) {
        /* [FFS] "Scale 怎样把 Tensor 塞进 E4M3": a_max over the tensor, one s, then the cast */
        j->s = orc_scale_from_amax(amax_all(j), fmt);
        ((float*)scale)[0] = j->s;
        orc_parallel(rows, 1, j, cast_rows);
    } else if (mode == ORC_ROW) {
        orc_parallel(rows, 1, j, row_rows);
    } else if (mode == ORC_BLOCK_1x128) {
        orc_parallel(rows, 1, j, block1_rows);
    } else if (mode == ORC_BLOCK_128x128) {
        orc_parallel(cdiv(rows, 128), 1, j, block128_rows);
    } else {
        orc_parallel(rows, 1, j, mx_rows);
    }
    free(j);
    return rc;
}

/*
 * orc_delayed_step: one step t of delayed per-tensor scaling ([FFS] "Delayed Scaling").
 *   ring[len] holds the amax history (zero-initialised by the caller).
 *   t == 0: no history yet -> the scale comes from the current amax.
 *   t >= 1: s_t = max(max(ring), 1e-12f) / F_max.
 *   After quantizing, ring[t mod len] <- amax_t (raw amax of this step's input).
 *   *saturated receives the number of elements with |x / s_t| > F_max.
 *   *scale_out receives s_t.
 * A step whose input holds a NaN or Inf is refused (returns 1) and records nothing:
 * ring[t mod len] keeps its value, so that one bad step cannot set the scale of the
 * next len steps ([FFS] "数值验证看什么": non-finite values are monitored; a
 * history is only a window of the amax of valid steps).  The caller still counts
 * the step (the next one is t + 1).
 */
int orc_delayed_step(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int fmt,
                     float* ring, int32_t len, int64_t t, uint8_t* q, float* scale_out,
                     uint16_t* dequant, int64_t* saturated) {
    if (rows < 0 || cols < 0 || ld < cols || len <= 0 || t < 0) return 2;
    if (fmt != ORC_E4M3 && fmt != ORC_E5M2) return 2;
    qjob* j = (qjob*)calloc(1, sizeof(qjob));
    if (!j) return 2;
    j->x = x; j->rows = rows; j->cols = cols; j->ld = ld; j->fmt = fmt;
    j->q = q; j->dequant = dequant;
    if (check_finite(j)) {
        free(j);
        return 1;
    }
    float amax_t = amax_all(j);
    float s;
    if (t == 0) {
        s = orc_scale_from_amax(amax_t, fmt);
    } else {
        float h = 0.0f;
        for (int32_t i = 0; i < len; ++i) if (ring[i] > h) h = ring[i];
        s = orc_scale_from_amax(h, fmt);
    }
    j->s = s;
    int parts = orc_parallel(rows, 1, j, cast_rows);
    int64_t sat_total = 0;
    for (int k = 0; k < parts; ++k) sat_total += j->sat_part[k];
    *scale_out = s;
    if (saturated) *saturated = sat_total;
    ring[t % len] = amax_t;
    free(j);
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

/* Reference at a list of output points (m[i], n[i]); the points are split into
 * contiguous ranges over the threads (each with its own dequantised rows). */
typedef struct {
    const uint8_t *a, *b;
    const void *sa, *sb;
    int a_mode, fmt_a, b_mode, fmt_b;
    int64_t M, N, K;
    const int64_t *pm, *pn;
    double *y, *bound;
    int err_part[ORC_MAX_THREADS];
} pjob;

static void points_range(void* c, int64_t i0, int64_t i1, int part) {
    pjob* j = (pjob*)c;
    int64_t K = j->K;
    double* ra = (double*)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
    double* rb = (double*)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
    j->err_part[part] = 0;
    if (!ra || !rb) { free(ra); free(rb); j->err_part[part] = 1; return; }
    int64_t cur_m = -1;
    for (int64_t i = i0; i < i1; ++i) {
        int64_t m = j->pm[i], n = j->pn[i];
        if (m < 0 || m >= j->M || n < 0 || n >= j->N) { j->err_part[part] = 1; break; }
        if (m != cur_m) { deq_row(j->a, j->sa, j->a_mode, j->fmt_a, m, K, ra); cur_m = m; }
        deq_row(j->b, j->sb, j->b_mode, j->fmt_b, n, K, rb);
        double acc = 0.0, bnd = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double p = ra[k] * rb[k];
            acc += p;
            bnd += fabs(p);
        }
        j->y[i] = acc;
        j->bound[i] = bnd;
    }
    free(ra);
    free(rb);
}

int orc_gemm_ref_points(const uint8_t* a, const void* sa, int a_mode, int fmt_a,
                        const uint8_t* b, const void* sb, int b_mode, int fmt_b,
                        int64_t M, int64_t N, int64_t K,
                        const int64_t* pm, const int64_t* pn, int64_t npts,
                        double* y, double* bound) {
    pjob* j = (pjob*)calloc(1, sizeof(pjob));
    if (!j) return 2;
    j->a = a; j->b = b; j->sa = sa; j->sb = sb;
    j->a_mode = a_mode; j->fmt_a = fmt_a; j->b_mode = b_mode; j->fmt_b = fmt_b;
    j->M = M; j->N = N; j->K = K; j->pm = pm; j->pn = pn; j->y = y; j->bound = bound;
    int parts = orc_parallel(npts, 1, j, points_range);
    int rc = 0;
    for (int k = 0; k < parts; ++k)
        if (j->err_part[k]) rc = 2;
    free(j);
    return rc;
}

/* Full reference: y and bound are [M, N]; rows of the output split over the threads. */
typedef struct {
    const double *da, *db;
    int64_t N, K;
    double *y, *bound;
} fjob;

static void full_rows(void* c, int64_t m0, int64_t m1, int part) {
    (void)part;
    fjob* j = (fjob*)c;
    for (int64_t m = m0; m < m1; ++m)
        for (int64_t n = 0; n < j->N; ++n) {
            double acc = 0.0, bnd = 0.0;
            for (int64_t k = 0; k < j->K; ++k) {
                double p = j->da[m * j->K + k] * j->db[n * j->K + k];
                acc += p;
                bnd += fabs(p);
            }
            j->y[m * j->N + n] = acc;
            j->bound[m * j->N + n] = bnd;
        }
}

int orc_gemm_ref_full(const uint8_t* a, const void* sa, int a_mode, int fmt_a,
                      const uint8_t* b, const void* sb, int b_mode, int fmt_b,
                      int64_t M, int64_t N, int64_t K, double* y, double* bound) {
    double* da = (double*)malloc(sizeof(double) * (size_t)(M * K > 0 ? M * K : 1));
    double* db = (double*)malloc(sizeof(double) * (size_t)(N * K > 0 ? N * K : 1));
    if (!da || !db) { free(da); free(db); return 2; }
    for (int64_t m = 0; m < M; ++m) deq_row(a, sa, a_mode, fmt_a, m, K, da + m * K);
    for (int64_t n = 0; n < N; ++n) deq_row(b, sb, b_mode, fmt_b, n, K, db + n * K);
    fjob j = {da, db, N, K, y, bound};
    orc_parallel(M, 1, &j, full_rows);
    free(da);
    free(db);
    return 0;
}

/* Whole output rows [m0, m1) x all N (y and bound are [m1 - m0, N]): the operand rows
 * of A are dequantised once; the N rows of B are split over the threads, each
 * dequantising one row of B at a time (memory stays at K doubles per thread). */
typedef struct {
    const uint8_t* b;
    const void* sb;
    int b_mode, fmt_b;
    const double* da;
    int64_t rows, N, K;
    double *y, *bound;
    int err_part[ORC_MAX_THREADS];
} rjob;

static void rows_range(void* c, int64_t n0, int64_t n1, int part) {
    rjob* j = (rjob*)c;
    double* rb = (double*)malloc(sizeof(double) * (size_t)(j->K > 0 ? j->K : 1));
    j->err_part[part] = rb == NULL;
    if (!rb) return;
    for (int64_t n = n0; n < n1; ++n) {
        deq_row(j->b, j->sb, j->b_mode, j->fmt_b, n, j->K, rb);
        for (int64_t i = 0; i < j->rows; ++i) {
            const double* ra = j->da + i * j->K;
            double acc = 0.0, bnd = 0.0;
            for (int64_t k = 0; k < j->K; ++k) {
                double p = ra[k] * rb[k];
                acc += p;
                bnd += fabs(p);
            }
            j->y[i * j->N + n] = acc;
            j->bound[i * j->N + n] = bnd;
        }
    }
    free(rb);
}

int orc_gemm_ref_slice(const uint8_t* a, const void* sa, int a_mode, int fmt_a,
                      const uint8_t* b, const void* sb, int b_mode, int fmt_b,
                      int64_t M, int64_t N, int64_t K, int64_t m0, int64_t m1,
                      double* y, double* bound) {
    if (m0 < 0 || m1 > M || m0 > m1) return 2;
    rjob* j = (rjob*)calloc(1, sizeof(rjob));
    double* da = (double*)malloc(sizeof(double) * (size_t)((m1 - m0) * K > 0 ? (m1 - m0) * K : 1));
    if (!j || !da) { free(j); free(da); return 2; }
    for (int64_t m = m0; m < m1; ++m) deq_row(a, sa, a_mode, fmt_a, m, K, da + (m - m0) * K);
    j->b = b; j->sb = sb; j->b_mode = b_mode; j->fmt_b = fmt_b; j->da = da;
    j->rows = m1 - m0; j->N = N; j->K = K; j->y = y; j->bound = bound;
    int parts = orc_parallel(N, 1, j, rows_range);
    int rc = 0;
    for (int k = 0; k < parts; ++k)
        if (j->err_part[k]) rc = 2;
    free(da);
    free(j);
    return rc;
}

/* Decoded values of every code of a format, for table-driven checks. */
void orc_decode_table(int fmt, double* out256) {
    for (int c = 0; c < 256; ++c) out256[c] = orc_decode((uint8_t)c, fmt);
}

/* Vector helpers so the tests can drive large arrays through ctypes. */
typedef struct {
    const float* v;
    float s;
    int fmt;
    uint8_t* out;
} ejob;
static void encode_range(void* c, int64_t i0, int64_t i1, int part) {
    const ejob* j = (const ejob*)c;
    (void)part;
    for (int64_t i = i0; i < i1; ++i) j->out[i] = orc_encode((double)j->v[i], j->fmt);
}
static void quant_scaled_range(void* c, int64_t i0, int64_t i1, int part) {
    const ejob* j = (const ejob*)c;
    (void)part;
    for (int64_t i = i0; i < i1; ++i) j->out[i] = quant_one(j->v[i], j->s, j->fmt, NULL);
}
void orc_encode_array(const float* v, int64_t n, int fmt, uint8_t* out) {
    ejob j = {v, 1.0f, fmt, out};
    orc_parallel(n, 4096, &j, encode_range);
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
    ejob j = {v, s, fmt, out};
    orc_parallel(n, 4096, &j, quant_scaled_range);
}
