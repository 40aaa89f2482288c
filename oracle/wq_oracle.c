/*
 * wq_oracle.c -- plain, slow, obviously-correct CPU oracle for group-wise RTN
 * affine weight quantization, dequantization and the W4A16 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path and includes no CUDA header.
 *
 * Sources (page title, section):
 *  [P1] "LLM Quantization: GPTQ, AWQ, SmoothQuant, FP8, KV Cache (7/10)",
 *       blog.ruahverce.com -- sections "Affine Quantization", "Bit count and
 *       level count", "Symmetric and Asymmetric", "Per-group", "Memory
 *       arithmetic: payload and metadata", "Group scale overhead",
 *       "Fused low-bit kernel (path A) / full dequantize then matmul (path B)".
 *  [P2] "Quantization Algorithms" (V10 study notes), brianyu43.github.io --
 *       section 1.8 "Signed vs Unsigned" (INT8 symmetric uses [-127,127],
 *       INT4 signed [-8,7], asymmetric unsigned [0,15]); "Fake vs real quant"
 *       section 4 (dequantized value multiplied in floating point, one
 *       rounding).
 *
 * What is computed (each step in the order the pages give it):
 *   quantize  q = clamp(round(x / s) + z, q_min, q_max)          [P1 Affine]
 *   symmetric z = 0, s = max|x| / q_max                          [P1 Symmetric]
 *   asymmetric s = (x_max - x_min) / (q_max - q_min),
 *              z = q_min - x_min / s, rounded and clamped so that
 *              zero is exactly representable                     [P1 Asymmetric]
 *   dequantize x_hat = s (q - z)                                 [P1 Affine]
 *   linear     y[m,n] = sum_k x_hat[n,k] * x[m,k]                [P1 path A/B]
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *   - round() is round-half-to-even, applied to the IEEE fp32 quotient x/s;
 *   - the quotient uses the STORED fp16 scale, so codes and dequant agree;
 *   - the asymmetric range is widened to contain 0 (x_min' = min(0, min x),
 *     x_max' = max(0, max x)) and z is an integer in [q_min, q_max]; then
 *     code z dequantizes to exactly 0;
 *   - s is computed in fp32 ((x_max' - x_min') / q_range, IEEE divide) and
 *     rounded to fp16 with round-to-nearest-even; a zero fp16 scale (all-zero
 *     or underflowing group) is replaced by s = 1, z = 0; an fp16 overflow
 *     saturates s to 65504 and raises WQO_FLAG_RANGE;
 *   - NaN inputs are skipped by the statistics and coded as the code of zero
 *     (q = z); any NaN/Inf input raises WQO_FLAG_NONFINITE;
 *   - symmetric 4-bit codes are stored as 4-bit two's complement nibbles;
 *   - packing: 8 nibbles per uint32, nibble j of word c holds column 8c+j
 *     (bits 4j..4j+3, low nibble first); scales/zeros are fp16 [d_out][d_in/g].
 *
 * Floating-point conversions are written here from the IEEE 754 definitions
 * (binary32 -> binary16 and binary32 -> bfloat16, round to nearest even,
 * subnormals included); nothing is taken from a vendor library.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* WQO_MUTANT (default 0) plants one deliberate mistake; the test suite
 * builds each mutant separately to show that the pins catch it.  The
 * shipped oracle is always built with WQO_MUTANT == 0. */
#ifndef WQO_MUTANT
#define WQO_MUTANT 0
#endif

#define WQO_FLAG_NONFINITE 1u
#define WQO_FLAG_RANGE 2u

/* ------------------------------------------------------------------------ */
/* IEEE 754 conversions                                                      */
/* ------------------------------------------------------------------------ */

static float bits_to_f32(uint32_t u) {
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static uint32_t f32_to_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

/* bfloat16 is the upper half of a binary32: widening is exact. */
float wqo_bf16_to_f32(uint16_t h) { return bits_to_f32((uint32_t)h << 16); }

/* binary32 -> bfloat16, round to nearest, ties to even.  The discarded low
 * 16 bits are compared with one half of the bf16 unit in the last place. */
uint16_t wqo_f32_to_bf16(float f) {
    uint32_t u = f32_to_bits(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) /* NaN: keep sign, force quiet */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xffffu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u)))
        kept += 1u; /* a carry into the exponent gives the next binade / inf */
    return (uint16_t)kept;
}

/* binary16 -> binary32, exact. */
float wqo_f16_to_f32(uint16_t h) {
    uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
    uint32_t e = (h >> 10) & 0x1fu;
    uint32_t m = h & 0x3ffu;
    if (e == 0x1fu) return bits_to_f32(sign | 0x7f800000u | (m << 13));
    if (e == 0) { /* zero or subnormal: m * 2^-24 */
        float v = (float)m * 0x1p-24f;
        return sign ? -v : v;
    }
    return bits_to_f32(sign | ((e - 15u + 127u) << 23) | (m << 13));
}

/* binary32 -> binary16, round to nearest, ties to even, with subnormals and
 * overflow to infinity.  Let the input be mant * 2^(e-23) with a 24-bit
 * integer significand.  The binary16 quantum at that magnitude is
 * 2^(max(e,-14) - 10); the number of quanta is mant >> sh with
 * sh = 13 + (max(e,-14) - e), rounded to nearest even on the dropped bits.
 * The encoding ((E + 14) << 10) + q is valid for normals and subnormals and
 * carries naturally into the next binade. */
uint16_t wqo_f32_to_f16(float f) {
    uint32_t u = f32_to_bits(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t a = u & 0x7fffffffu;
    if (a > 0x7f800000u) return (uint16_t)(sign | 0x7e00u); /* NaN */
    if (a == 0x7f800000u) return (uint16_t)(sign | 0x7c00u); /* inf */
    int e;
    uint32_t mant;
    if (a >= 0x00800000u) {
        e = (int)(a >> 23) - 127;
        mant = (a & 0x7fffffu) | 0x800000u;
    } else {
        e = -126;
        mant = a;
    }
    int E = e > -14 ? e : -14;
    int sh = 13 + (E - e);
    uint32_t q;
    if (sh >= 25) {
        q = 0; /* below half of the smallest subnormal */
    } else {
        q = mant >> sh;
        uint32_t rem = mant & ((1u << sh) - 1u);
        uint32_t half = 1u << (sh - 1);
        if (rem > half || (rem == half && (q & 1u))) q += 1u;
    }
    int64_t bits = ((int64_t)(E + 14) << 10) + (int64_t)q;
    if (bits >= 0x7c00) return (uint16_t)(sign | 0x7c00u);
    return (uint16_t)(sign | (uint16_t)bits);
}

/* ------------------------------------------------------------------------ */
/* Quantization parameters                                                   */
/* ------------------------------------------------------------------------ */

typedef struct {
    int bits;       /* b: 2, 4 or 8 */
    int symmetric;  /* 1: z = 0, signed codes */
    int narrow;     /* symmetric only: q_min = -q_max (INT8 [-127,127]) */
} wqo_qparams;

/* Code range: unsigned b bits give 2^b levels [0, 2^b - 1]; signed b bits
 * give [-2^(b-1), 2^(b-1) - 1], and the narrow symmetric form drops the
 * negative endpoint ([P1 Bit count and level count], [P2 1.8]). */
static void code_range(const wqo_qparams* p, int* qmin, int* qmax) {
    if (p->symmetric) {
        *qmax = (1 << (p->bits - 1)) - 1;
        *qmin = p->narrow ? -*qmax : -(1 << (p->bits - 1));
    } else {
        *qmin = 0;
        *qmax = (1 << p->bits) - 1;
    }
}

/* Clamp with IEEE maxNum/minNum semantics, then convert the (integral)
 * float to int.  Inputs here are never NaN. */
static int clamp_to_int(float v, int lo, int hi) {
    if (v < (float)lo) v = (float)lo;
    if (v > (float)hi) v = (float)hi;
    return (int)v;
}

/* Scale and zero point of a group whose range is [lo, hi] (asymmetric, lo <= 0
 * <= hi) or [-amax, amax] (symmetric); then the codes of its g weights.
 * Returns WQO_FLAG_RANGE if the fp16 scale saturated. */
static uint32_t quantize_with_range(const uint16_t* x, int64_t g, const wqo_qparams* p, float lo,
                                    float hi, float amax, int32_t* codes, uint16_t* s_out,
                                    int* z_out) {
    int qmin, qmax;
    code_range(p, &qmin, &qmax);
    uint32_t flags = 0;

    /* scale in fp32, stored as fp16 */
    float s32;
    if (p->symmetric)
#if WQO_MUTANT == 15 /* mistake: symmetric scale over 2^(b-1) instead of 2^(b-1) - 1 */
        s32 = amax / (float)(-qmin);
#else
        s32 = amax / (float)qmax;
#endif
    else
#if WQO_MUTANT == 3 /* mistake: divide by the level count, not the range */
        s32 = (hi - lo) / (float)(qmax - qmin + 1);
#else
        s32 = (hi - lo) / (float)(qmax - qmin);
#endif
    uint16_t s16 = wqo_f32_to_f16(s32);
    int z = 0;
    if (s16 == 0x7c00u) { /* fp16 overflow: saturate */
        s16 = 0x7bffu;
        flags |= WQO_FLAG_RANGE;
    }
    if (s16 == 0x0000u) { /* all-zero or underflowing group */
        s16 = 0x3c00u;  /* 1.0 */
        z = 0;
    } else if (!p->symmetric) {
        float s = wqo_f16_to_f32(s16);
        /* z = q_min - x_min/s, rounded (half to even) and clamped */
#if WQO_MUTANT == 1 /* mistake: wrong sign of the zero point */
        float zf = rintf((float)qmin + lo / s);
#else
        float zf = rintf((float)qmin - lo / s);
#endif
        z = clamp_to_int(zf, qmin, qmax);
    }
    float s = wqo_f16_to_f32(s16);

    /* codes [P1 Affine]: q = clamp(round(x/s) + z, q_min, q_max) */
    for (int64_t k = 0; k < g; ++k) {
        float v = wqo_bf16_to_f32(x[k]);
        if (isnan(v)) {
#if WQO_MUTANT == 17 /* mistake: NaN takes the lowest code instead of the code of zero */
            codes[k] = qmin;
#else
            codes[k] = z; /* NaN is coded as zero */
#endif
            continue;
        }
#if WQO_MUTANT == 2 /* mistake: round half away from zero */
        float t = roundf(v / s);
#else
        float t = rintf(v / s);
#endif
        codes[k] = clamp_to_int(t + (float)z, qmin, qmax);
    }
    *s_out = s16;
    *z_out = z;
    return flags;
}

/* One group: derive (s, z) and the codes of g consecutive weights of one row.
 * x: g bf16 words; codes: g ints; returns flags. */
static uint32_t quantize_group(const uint16_t* x, int64_t g, const wqo_qparams* p,
                               int32_t* codes, uint16_t* s_out, uint16_t* z_out) {
    uint32_t flags = 0;

    /* statistics [P1 Symmetric / Asymmetric]; range widened to contain 0 */
    float lo = 0.0f, hi = 0.0f, amax = 0.0f;
#if WQO_MUTANT == 4 /* mistake: range not widened to contain zero */
    lo = INFINITY;
    hi = -INFINITY;
#endif
    for (int64_t k = 0; k < g; ++k) {
        float v = wqo_bf16_to_f32(x[k]);
        if (!isfinite(v)) flags |= WQO_FLAG_NONFINITE;
        if (isnan(v)) continue;
        if (v < lo) lo = v;
        if (v > hi) hi = v;
        float av = fabsf(v);
        if (av > amax) amax = av;
    }

    int z;
    flags |= quantize_with_range(x, g, p, lo, hi, amax, codes, s_out, &z);
    if (z_out) *z_out = wqo_f32_to_f16((float)z);
    return flags;
}

/* ------------------------------------------------------------------------ */
/* Row-parallel driver (pthreads over row ranges; the per-row code is the    */
/* plain loop above).                                                        */
/* ------------------------------------------------------------------------ */

typedef void (*row_fn)(void* ctx, int64_t r0, int64_t r1, uint32_t* flags);

typedef struct {
    row_fn fn;
    void* ctx;
    int64_t r0, r1;
    uint32_t flags;
} row_job;

static void* row_job_main(void* arg) {
    row_job* j = (row_job*)arg;
    j->flags = 0;
    j->fn(j->ctx, j->r0, j->r1, &j->flags);
    return NULL;
}

static uint32_t run_rows(row_fn fn, void* ctx, int64_t rows, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads > rows) nthreads = rows > 0 ? (int)rows : 1;
    row_job jobs[256];
    pthread_t tids[256];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].fn = fn;
        jobs[t].ctx = ctx;
        jobs[t].r0 = rows * t / nthreads;
        jobs[t].r1 = rows * (t + 1) / nthreads;
    }
    for (int t = 1; t < nthreads; ++t) pthread_create(&tids[t], NULL, row_job_main, &jobs[t]);
    row_job_main(&jobs[0]);
    uint32_t flags = jobs[0].flags;
    for (int t = 1; t < nthreads; ++t) {
        pthread_join(tids[t], NULL);
        flags |= jobs[t].flags;
    }
    return flags;
}

/* ------------------------------------------------------------------------ */
/* Quantize                                                                  */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t* W;
    int64_t d_in, g;
    wqo_qparams p;
    int32_t* codes;
    uint16_t* scales;
    uint16_t* zeros;
} quant_ctx;

static void quant_rows(void* vctx, int64_t r0, int64_t r1, uint32_t* flags) {
    quant_ctx* c = (quant_ctx*)vctx;
    int64_t ng = c->d_in / c->g;
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t j = 0; j < ng; ++j) {
            int64_t off = r * c->d_in + j * c->g;
            *flags |= quantize_group(c->W + off, c->g, &c->p, c->codes + off,
                                     c->scales + r * ng + j,
                                     c->zeros ? c->zeros + r * ng + j : NULL);
        }
}

/* W: bf16 bits [d_out][d_in]; codes: int32 [d_out][d_in];
 * scales, zeros: fp16 bits [d_out][d_in/g] (zeros may be NULL when symmetric).
 * Returns 0 on success, -1 on bad arguments; *flags gets WQO_FLAG_*. */
int wqo_quantize(const uint16_t* W, int64_t d_out, int64_t d_in, int64_t g, int bits,
                 int symmetric, int narrow, int32_t* codes, uint16_t* scales,
                 uint16_t* zeros, uint32_t* flags, int nthreads) {
    if (!W || !codes || !scales || d_out < 0 || d_in <= 0 || g <= 0 || d_in % g != 0)
        return -1;
    if (bits < 2 || bits > 8) return -1;
    if (!symmetric && !zeros) return -1;
    quant_ctx c = {W, d_in, g, {bits, symmetric, narrow}, codes, scales, symmetric ? NULL : zeros};
    uint32_t f = run_rows(quant_rows, &c, d_out, nthreads);
    if (flags) *flags = f;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* MSE-optimal clipping per group                                            */
/* [P1 Clipping Trade-off]: a range set by one large value coarsens every    */
/* level; clipping it trades that value's error for the rest's.  The         */
/* threshold is chosen to minimise the local reconstruction error            */
/* [P2 calibration section 4: MSE-optimal, argmin ||x - x_dq||^2, chosen per  */
/* channel/group independently].                                             */
/* Readings (the pages give no grid or summation order):                     */
/*  - candidates shrink the RTN range by alpha_i = fl32((20 - i) / 20),      */
/*    i = 0..10 (1.00, 0.95, ..., 0.50): lo_i = fl32(alpha_i lo),             */
/*    hi_i = fl32(alpha_i hi) (amax_i likewise); scale, zero and codes follow */
/*    the RTN formulas on that range, values outside it are clamped by the    */
/*    code range;                                                            */
/*  - the error is sum_k (x_k - x_hat_k)^2 over the finite x_k, x_hat_k the   */
/*    bf16 dequantized value, in fp64: the difference, its square rounded     */
/*    once, then the add (no fused multiply-add); the sum runs over runs of 8  */
/*    consecutive weights in order, then a pairwise tree over the runs in     */
/*    index order (g/8 must be a power of two);                               */
/*  - the smallest error wins; ties go to the smaller i (less clipping).      */
/* alpha_0 = 1 is plain RTN, so the chosen error never exceeds RTN's.        */
/* ------------------------------------------------------------------------ */

#define WQO_CLIP_CANDIDATES 11

uint16_t wqo_dequant_one(uint16_t s16, int32_t q, int32_t z);

/* One group quantized on a given range (test access to the candidate step). */
uint32_t wqo_quantize_group_range(const uint16_t* x, int64_t g, int bits, int symmetric, float lo,
                                  float hi, float amax, int32_t* codes, uint16_t* s16, int32_t* z) {
    wqo_qparams p = {bits, symmetric, 0};
    int zi;
    uint32_t f = quantize_with_range(x, g, &p, lo, hi, amax, codes, s16, &zi);
    *z = zi;
    return f;
}

float wqo_clip_alpha(int i) { return (float)(20 - i) / 20.0f; }

/* Squared reconstruction error of one group in the order stated above. */
double wqo_group_sq_error(const uint16_t* x, int64_t g, const int32_t* codes, uint16_t s16, int z) {
    int64_t runs = g / 8;
    double part[512];
    for (int64_t r = 0; r < runs; ++r) {
        double acc = 0.0;
        for (int64_t k = 8 * r; k < 8 * r + 8; ++k) {
            float v = wqo_bf16_to_f32(x[k]);
            if (!isfinite(v)) continue;
            double xh = (double)wqo_bf16_to_f32(wqo_dequant_one(s16, codes[k], z));
#if WQO_MUTANT == 9 /* mistake: absolute error instead of its square */
            double e = fabs((double)v - xh);
#else
            double e = ((double)v - xh) * ((double)v - xh);
#endif
            acc += e;
        }
        part[r] = acc;
    }
    for (int64_t w = 1; w < runs; w *= 2)
        for (int64_t r = 0; r + w < runs; r += 2 * w) part[r] = part[r] + part[r + w];
    return part[0];
}

/* One group with the clipping search; *best gets the chosen candidate index. */
static uint32_t quantize_group_clip(const uint16_t* x, int64_t g, const wqo_qparams* p,
                                    int32_t* codes, uint16_t* s_out, uint16_t* z_out,
                                    uint8_t* best) {
    uint32_t flags = 0;
    float lo = 0.0f, hi = 0.0f, amax = 0.0f;
    for (int64_t k = 0; k < g; ++k) {
        float v = wqo_bf16_to_f32(x[k]);
        if (!isfinite(v)) flags |= WQO_FLAG_NONFINITE;
        if (isnan(v)) continue;
        if (v < lo) lo = v;
        if (v > hi) hi = v;
        float av = fabsf(v);
        if (av > amax) amax = av;
    }
    int32_t cand[1024];
    double best_err = 0.0;
    int best_i = -1, best_z = 0;
    uint16_t best_s = 0;
    uint32_t best_flags = 0;
    for (int i = 0; i < WQO_CLIP_CANDIDATES; ++i) {
        float a = wqo_clip_alpha(i);
        uint16_t s16;
        int z;
#if WQO_MUTANT == 20 /* mistake: only the upper end of the range is shrunk */
        uint32_t f = quantize_with_range(x, g, p, lo, a * hi, a * amax, cand, &s16, &z);
#else
        uint32_t f = quantize_with_range(x, g, p, a * lo, a * hi, a * amax, cand, &s16, &z);
#endif
        double err = wqo_group_sq_error(x, g, cand, s16, z);
#if WQO_MUTANT == 10 /* mistake: the largest error wins */
        if (best_i < 0 || err > best_err) {
#else
        if (best_i < 0 || err < best_err) {
#endif
            best_i = i;
            best_err = err;
            best_s = s16;
            best_z = z;
            best_flags = f;
            for (int64_t k = 0; k < g; ++k) codes[k] = cand[k];
        }
    }
    *s_out = best_s;
    if (z_out) *z_out = wqo_f32_to_f16((float)best_z);
    if (best) *best = (uint8_t)best_i;
    return flags | best_flags;
}

typedef struct {
    const uint16_t* W;
    int64_t d_in, g;
    wqo_qparams p;
    int32_t* codes;
    uint16_t* scales;
    uint16_t* zeros;
    uint8_t* best;
} clip_ctx;

static void clip_rows(void* vctx, int64_t r0, int64_t r1, uint32_t* flags) {
    clip_ctx* c = (clip_ctx*)vctx;
    int64_t ng = c->d_in / c->g;
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t j = 0; j < ng; ++j) {
            int64_t off = r * c->d_in + j * c->g;
            *flags |= quantize_group_clip(c->W + off, c->g, &c->p, c->codes + off, c->scales + r * ng + j,
                                          c->zeros ? c->zeros + r * ng + j : NULL,
                                          c->best ? c->best + r * ng + j : NULL);
        }
}

/* As wqo_quantize, with the clipping search; best: chosen candidate index per
 * group [d_out][d_in/g] (may be NULL).  g/8 must be a power of two, g <= 1024. */
int wqo_quantize_clip(const uint16_t* W, int64_t d_out, int64_t d_in, int64_t g, int bits,
                      int symmetric, int32_t* codes, uint16_t* scales, uint16_t* zeros,
                      uint8_t* best, uint32_t* flags, int nthreads) {
    if (!W || !codes || !scales || d_out < 0 || d_in <= 0 || g < 8 || g > 1024 || d_in % g != 0) return -1;
    if ((g % 8) != 0 || ((g / 8) & (g / 8 - 1)) != 0) return -1;
    if (bits < 2 || bits > 8) return -1;
    if (!symmetric && !zeros) return -1;
    clip_ctx c = {W, d_in, g, {bits, symmetric, 0}, codes, scales, symmetric ? NULL : zeros, best};
    uint32_t f = run_rows(clip_rows, &c, d_out, nthreads);
    if (flags) *flags = f;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* AWQ: activation-aware per-input-channel scaling                           */
/* [P2 "AWQ" procedure]: per-channel mean |x| over a calibration batch; for   */
/* alpha in {0, 0.1, ..., 1.0}: s = mean|x|^alpha / geomean, W' = W diag(s),  */
/* loss = ||W X - Q(W') (X / s)||; keep the argmin; s^-1 is fused into the    */
/* previous layer [P1 "AWQ": protect salient channels found from activation   */
/* statistics through per-channel scaling].                                  */
/* Readings (the pages leave them open):                                     */
/*  - m_j = (sum_t |X[t,j]|) / T in fp64 (exact sum of bf16 values), floored  */
/*    at 2^-30;                                                              */
/*  - alpha_i = i / 10 (fp64), i = 0..10;                                     */
/*  - s_j = bf16_rn(fl32(exp(alpha (ln m_j - mean_j ln m_j)))), i.e. m^alpha  */
/*    over its geometric mean (fp64), rounded to fp32 then bf16, so that the  */
/*    two products below are one multiply or divide and one rounding each;    */
/*    ln and exp are wqo_ln_f64 / wqo_exp_f64 below (a fixed fp64 procedure), */
/*    the mean of ln m is summed in channel order;                            */
/*  - W'[n,j] = bf16_rn(fl32(W[n,j] s_j)); X'[t,j] = bf16_rn(fl32(X[t,j]/s_j)); */
/*  - Q(W') is the RTN artifact of W' (quantize_group) and its dequant;        */
/*  - loss = sum_{t,n} (Y[t,n] - Y'[t,n])^2 with Y = X W^T and Y' = X' Q(W')^T  */
/*    in fp64; the smallest loss wins, ties to the smaller alpha.             */
/* alpha = 0 gives s = 1, i.e. plain RTN of W.                                */
/* ------------------------------------------------------------------------ */

#define WQO_AWQ_ALPHAS 11

/* ln and exp of the AWQ scales, as one fixed sequence of IEEE binary64       */
/* operations (each multiply, add, subtract and divide rounded on its own, no */
/* fused multiply-add: this file is compiled with -ffp-contract=off), so that */
/* any implementation that follows the same steps obtains the same bits; the  */
/* pages give the formula s = m^alpha / geomean but no evaluation procedure.  */
/* Both use the argument reduction of W. J. Cody and W. Waite, "Software      */
/* Manual for the Elementary Functions" (1980): ln 2 split into a head with   */
/* 21 trailing zero bits (k ln2_hi exact for |k| < 2^21) and a tail.          */
static const double WQO_LN2_HI = 0x1.62e42fee00000p-1;
static const double WQO_LN2_LO = 0x1.a39ef35793c76p-33;
static const double WQO_INV_LN2 = 0x1.71547652b82fep+0;
static const double WQO_SQRT2 = 0x1.6a09e667f3bcdp+0;

/* ln x for a positive normal x: x = f 2^e with f in [sqrt(2)/2, sqrt(2)),     */
/* u = (f - 1) / (f + 1), ln f = 2 atanh u = 2 u (1 + u^2/3 + u^4/5 + ...),    */
/* twelve terms (|u| <= 0.1716, the first dropped term is below 2^-60),       */
/* evaluated by Horner's rule in u^2; ln x = e ln2_hi + (e ln2_lo + ln f).     */
double wqo_ln_f64(double x) {
    uint64_t b;
    memcpy(&b, &x, 8);
    int e = (int)((b >> 52) & 0x7ff) - 1023;
    const uint64_t fb = (b & 0x000fffffffffffffull) | 0x3ff0000000000000ull;
    double f;
    memcpy(&f, &fb, 8);
    if (f > WQO_SQRT2) {
        f = f * 0.5;
        e += 1;
    }
    const double u = (f - 1.0) / (f + 1.0);
    const double v = u * u;
    double p = 1.0 / 23.0;
    for (int k = 10; k >= 0; --k) p = p * v + 1.0 / (double)(2 * k + 1);
    const double lnf = (u + u) * p;
    const double de = (double)e;
    return de * WQO_LN2_HI + (de * WQO_LN2_LO + lnf);
}

/* e^x for |x| < 700: k = rint(x / ln 2) (round half to even, by adding and   */
/* subtracting 1.5 2^52), r = (x - k ln2_hi) - k ln2_lo, e^r by its Taylor    */
/* polynomial of degree 13 (|r| <= 0.347, the first dropped term below 2^-57) */
/* in Horner form with coefficients 1/i!, then the exact product by 2^k.      */
double wqo_exp_f64(double x) {
    const double magic = 0x1.8p52;
    const double kd = (x * WQO_INV_LN2 + magic) - magic;
    const double r = (x - kd * WQO_LN2_HI) - kd * WQO_LN2_LO;
    double fact = 1.0;
    for (int i = 2; i <= 13; ++i) fact *= (double)i;  /* 13!, exact */
    double p = 1.0 / fact;
    for (int i = 12; i >= 0; --i) {
        fact /= (double)(i + 1);                       /* i!, exact */
        p = p * r + 1.0 / fact;
    }
    const uint64_t sb = (uint64_t)((int64_t)kd + 1023) << 52;
    double scale;
    memcpy(&scale, &sb, 8);
    return p * scale;
}

int wqo_dequantize(const int32_t* codes, const uint16_t* scales, const uint16_t* zeros, int64_t d_out,
                   int64_t d_in, int64_t g, uint16_t* W_hat, int nthreads);

/* Y[t][n] = sum_j A[t][j] B[n][j] in fp64 for bf16 inputs (rows of A: T, rows of B: N). */
typedef struct {
    const uint16_t *A, *B;
    int64_t T, N, K;
    double* Y;
} gemm_ctx;

static void gemm_rows(void* vctx, int64_t t0, int64_t t1, uint32_t* flags) {
    gemm_ctx* c = (gemm_ctx*)vctx;
    (void)flags;
    for (int64_t t = t0; t < t1; ++t)
        for (int64_t n = 0; n < c->N; ++n) {
            double acc = 0.0;
            for (int64_t j = 0; j < c->K; ++j)
                acc += (double)wqo_bf16_to_f32(c->A[t * c->K + j]) * (double)wqo_bf16_to_f32(c->B[n * c->K + j]);
            c->Y[t * c->N + n] = acc;
        }
}

static void gemm_bf16_f64(const uint16_t* A, int64_t T, const uint16_t* B, int64_t N, int64_t K, double* Y,
                          int nthreads) {
    gemm_ctx c = {A, B, T, N, K, Y};
    run_rows(gemm_rows, &c, T, nthreads);
}

/* Per-channel scales for one alpha (bf16 bits). */
void wqo_awq_scales(const uint16_t* X, int64_t T, int64_t K, double alpha, uint16_t* s_out) {
    double* lnm = (double*)malloc(sizeof(double) * (size_t)K);
    double mean_ln = 0.0;
    for (int64_t j = 0; j < K; ++j) {
        double acc = 0.0;
        for (int64_t t = 0; t < T; ++t) acc += fabs((double)wqo_bf16_to_f32(X[t * K + j]));
        double m = acc / (double)T;
        if (m < 0x1p-30) m = 0x1p-30;
        lnm[j] = wqo_ln_f64(m);
    }
    for (int64_t j = 0; j < K; ++j) mean_ln += lnm[j];
    mean_ln /= (double)K;
    for (int64_t j = 0; j < K; ++j) {
#if WQO_MUTANT == 11 /* mistake: scales inverted (divide instead of multiply) */
        s_out[j] = wqo_f32_to_bf16((float)wqo_exp_f64(-alpha * (lnm[j] - mean_ln)));
#elif WQO_MUTANT == 19 /* mistake: not normalised by the geometric mean */
        s_out[j] = wqo_f32_to_bf16((float)wqo_exp_f64(alpha * lnm[j]));
#else
        s_out[j] = wqo_f32_to_bf16((float)wqo_exp_f64(alpha * (lnm[j] - mean_ln)));
#endif
    }
    free(lnm);
}

/* Search; outputs the artifact of the best alpha, its scales s (bf16 [K]),
 * the 11 losses and the best index.  Returns 0, or -1 on bad arguments. */
int wqo_awq_search(const uint16_t* W, int64_t N, int64_t K, const uint16_t* X, int64_t T, int64_t g,
                   int symmetric, int32_t* codes, uint16_t* scales, uint16_t* zeros, uint16_t* s_best,
                   double* losses, int32_t* best, int nthreads) {
    if (!W || !X || !codes || !scales || !s_best || N < 1 || K < 1 || T < 1 || g < 1 || K % g != 0) return -1;
    if (!symmetric && !zeros) return -1;
    const int64_t G = K / g;
    uint16_t* s = (uint16_t*)malloc(2 * (size_t)K);
    uint16_t* Wp = (uint16_t*)malloc(2 * (size_t)(N * K));
    uint16_t* Xp = (uint16_t*)malloc(2 * (size_t)(T * K));
    uint16_t* Wh = (uint16_t*)malloc(2 * (size_t)(N * K));
    int32_t* cc = (int32_t*)malloc(4 * (size_t)(N * K));
    uint16_t* sc = (uint16_t*)malloc(2 * (size_t)(N * G));
    uint16_t* zc = (uint16_t*)malloc(2 * (size_t)(N * G));
    double* Y = (double*)malloc(sizeof(double) * (size_t)(T * N));
    double* Yp = (double*)malloc(sizeof(double) * (size_t)(T * N));
    gemm_bf16_f64(X, T, W, N, K, Y, nthreads);
    double best_loss = 0.0;
    int best_i = -1;
    for (int i = 0; i < WQO_AWQ_ALPHAS; ++i) {
        double alpha = (double)i / 10.0;
        wqo_awq_scales(X, T, K, alpha, s);
        for (int64_t n = 0; n < N; ++n)
            for (int64_t j = 0; j < K; ++j)
                Wp[n * K + j] = wqo_f32_to_bf16(wqo_bf16_to_f32(W[n * K + j]) * wqo_bf16_to_f32(s[j]));
        for (int64_t t = 0; t < T; ++t)
            for (int64_t j = 0; j < K; ++j)
#if WQO_MUTANT == 21 /* mistake: activations multiplied by s instead of divided */
                Xp[t * K + j] = wqo_f32_to_bf16(wqo_bf16_to_f32(X[t * K + j]) * wqo_bf16_to_f32(s[j]));
#else
                Xp[t * K + j] = wqo_f32_to_bf16(wqo_bf16_to_f32(X[t * K + j]) / wqo_bf16_to_f32(s[j]));
#endif
        uint32_t fl;
        wqo_quantize(Wp, N, K, g, 4, symmetric, 0, cc, sc, symmetric ? NULL : zc, &fl, nthreads);
        wqo_dequantize(cc, sc, symmetric ? NULL : zc, N, K, g, Wh, nthreads);
        gemm_bf16_f64(Xp, T, Wh, N, K, Yp, nthreads);
        double loss = 0.0;
        for (int64_t q = 0; q < T * N; ++q) {
            double d = Y[q] - Yp[q];
            loss += d * d;
        }
        if (losses) losses[i] = loss;
        if (best_i < 0 || loss < best_loss) {
            best_i = i;
            best_loss = loss;
            for (int64_t q = 0; q < N * K; ++q) codes[q] = cc[q];
            for (int64_t q = 0; q < N * G; ++q) scales[q] = sc[q];
            if (!symmetric)
                for (int64_t q = 0; q < N * G; ++q) zeros[q] = zc[q];
            for (int64_t j = 0; j < K; ++j) s_best[j] = s[j];
        }
    }
    if (best) *best = best_i;
    free(s); free(Wp); free(Xp); free(Wh); free(cc); free(sc); free(zc); free(Y); free(Yp);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* GPTQ: error feedback through the inverse Hessian.                          */
/* [P2] "Quantization Algorithms" study notes, GPTQ chapter: layer-wise       */
/* objective ||W X - W_hat X||^2; Hessian H = 2 X X^T with a 1 % dampening of  */
/* the diagonal; the factor L = Cholesky(H^-1); columns quantized one at a    */
/* time in blocks of 128 -- err = (w_j - q_j) / L[j][j], the later columns of  */
/* the block updated with err L[j][.], the columns after the block updated    */
/* with the block's errors at once; settings W4, group 128, symmetric,        */
/* act-order on (columns with large |x|^2 first), damp 0.01.                  */
/* [P1] GPTQ section: one-shot PTQ that corrects the effect of each weight's   */
/* quantization error on the layer output.                                   */
/* Readings (the pages leave these open):                                    */
/*  - X is [T][K] (tokens x input channels), so H = 2 X^T X is K x K;          */
/*    H[a][b] = 2 sum_t x[t][a] x[t][b], summed in t order;                    */
/*  - dampening adds d = 0.01 mean(diag H) (diagonal summed in index order)    */
/*    to every diagonal entry; d = 1 when that mean is 0 (no signal at all);   */
/*  - act-order: columns are processed by decreasing damped H[j][j], ties in   */
/*    index order; the permutation applies to H's rows and columns and to W's  */
/*    columns; without act-order the order is the identity;                   */
/*  - "Cholesky(H^-1)" is the upper-triangular U with H^-1 = U^T U (the update */
/*    reads row j of the factor right of the diagonal); H^-1 = Linv^T Linv     */
/*    with Linv the inverse of the lower Cholesky factor of H;                */
/*  - quant() is the layer's group-wise quantizer with STATIC parameters: the  */
/*    scale and zero point of each group of g input channels are plain RTN's   */
/*    on the original W (the artifact keeps contiguous groups, with or without */
/*    act-order); a code is clamp(rint(w / s) + z) with w / s the IEEE fp64     */
/*    quotient of the current weight, and the quantized value is              */
/*    bf16_rn(s (q - z)), the weight the W4A16 layer multiplies by;           */
/*  - fp64 throughout, every product rounded before its add or subtract (no    */
/*    fused multiply-add), sums in ascending index order:                    */
/*      Cholesky: a[i][j] - l[i][0] l[j][0] - l[i][1] l[j][1] - ... in turn,   */
/*      then divided by l[j][j] (the diagonal: its square root);              */
/*      Linv by forward substitution: v = sum_{k=j}^{i-1} l[i][k] Linv[k][j],  */
/*      Linv[i][j] = -v / l[i][i], Linv[j][j] = 1 / l[j][j];                   */
/*      H^-1[i][j] = sum_{k >= max(i,j)} Linv[k][i] Linv[k][j];               */
/*      U by the same Cholesky on H^-1 (U[i][j] = the lower factor's [j][i]);  */
/*      block tail: acc = sum_{j in block} err_j U[j][k], then w_k -= acc;     */
/*  - a Cholesky pivot that is not positive and finite (non-finite or          */
/*    numerically singular input) is replaced by 1 and raises WQO_FLAG_RANGE. */
/* ------------------------------------------------------------------------ */

#define WQO_GPTQ_BLOCK 128

typedef struct {
    const uint16_t* X;
    int64_t T, K;
    double* H;
} hess_ctx;

static void hess_rows(void* vctx, int64_t a0, int64_t a1, uint32_t* flags) {
    hess_ctx* c = (hess_ctx*)vctx;
    (void)flags;
    for (int64_t a = a0; a < a1; ++a)
        for (int64_t b = 0; b < c->K; ++b) {
            double acc = 0.0;
            for (int64_t t = 0; t < c->T; ++t)
                acc += (double)wqo_bf16_to_f32(c->X[t * c->K + a]) * (double)wqo_bf16_to_f32(c->X[t * c->K + b]);
            c->H[a * c->K + b] = 2.0 * acc;
        }
}

/* Lower Cholesky factor of the symmetric A (K x K, row-major), in place in
 * the lower triangle of L (the strict upper triangle is zeroed). */
typedef struct {
    double* L;
    int64_t K, j;
} chol_ctx;

static void chol_col_rows(void* vctx, int64_t r0, int64_t r1, uint32_t* flags) {
    chol_ctx* c = (chol_ctx*)vctx;
    (void)flags;
    const int64_t K = c->K, j = c->j;
    const double ljj = c->L[j * K + j];
    for (int64_t i = j + 1 + r0; i < j + 1 + r1; ++i) {
        double v = c->L[i * K + j];
        for (int64_t k = 0; k < j; ++k) v = v - c->L[i * K + k] * c->L[j * K + k];
        c->L[i * K + j] = v / ljj;
    }
}

static uint32_t cholesky_lower(const double* A, double* L, int64_t K, int nthreads) {
    uint32_t flags = 0;
    for (int64_t i = 0; i < K; ++i)
        for (int64_t j = 0; j < K; ++j) L[i * K + j] = j <= i ? A[i * K + j] : 0.0;
    for (int64_t j = 0; j < K; ++j) {
        double d = L[j * K + j];
        for (int64_t k = 0; k < j; ++k) d = d - L[j * K + k] * L[j * K + k];
        if (!(d > 0.0) || !isfinite(d)) {
            d = 1.0;
            flags |= WQO_FLAG_RANGE;
        }
        L[j * K + j] = sqrt(d);
        chol_ctx c = {L, K, j};
        if (K - j - 1 > 0) run_rows(chol_col_rows, &c, K - j - 1, (K - j - 1) >= 256 ? nthreads : 1);
    }
    return flags;
}

/* Linv = L^-1 by forward substitution, one column j per unit of work. */
typedef struct {
    const double* L;
    double* Li;
    int64_t K;
} trinv_ctx;

static void trinv_cols(void* vctx, int64_t j0, int64_t j1, uint32_t* flags) {
    trinv_ctx* c = (trinv_ctx*)vctx;
    (void)flags;
    const int64_t K = c->K;
    for (int64_t j = j0; j < j1; ++j) {
        for (int64_t i = 0; i < j; ++i) c->Li[i * K + j] = 0.0;
        c->Li[j * K + j] = 1.0 / c->L[j * K + j];
        for (int64_t i = j + 1; i < K; ++i) {
            double v = 0.0;
            for (int64_t k = j; k < i; ++k) v = v + c->L[i * K + k] * c->Li[k * K + j];
            c->Li[i * K + j] = -v / c->L[i * K + i];
        }
    }
}

/* Hinv[i][j] = sum_{k >= max(i,j)} Linv[k][i] Linv[k][j]. */
typedef struct {
    const double* Li;
    double* Hi;
    int64_t K;
} gram_ctx;

static void gram_rows(void* vctx, int64_t i0, int64_t i1, uint32_t* flags) {
    gram_ctx* c = (gram_ctx*)vctx;
    (void)flags;
    const int64_t K = c->K;
    for (int64_t i = i0; i < i1; ++i)
        for (int64_t j = 0; j < K; ++j) {
            double acc = 0.0;
            for (int64_t k = i > j ? i : j; k < K; ++k) acc = acc + c->Li[k * K + i] * c->Li[k * K + j];
            c->Hi[i * K + j] = acc;
        }
}

/* The factor U (upper, U^T U = H^-1) of the column-permuted damped Hessian
 * of X; perm[p] is the input channel processed p-th.  U: K x K row-major. */
uint32_t wqo_gptq_factor(const uint16_t* X, int64_t T, int64_t K, int act_order, int32_t* perm, double* U,
                         int nthreads) {
    uint32_t flags = 0;
    double* H = (double*)malloc(sizeof(double) * (size_t)(K * K));
    double* Hp = (double*)malloc(sizeof(double) * (size_t)(K * K));
    double* L = (double*)malloc(sizeof(double) * (size_t)(K * K));
    hess_ctx hc = {X, T, K, H};
    run_rows(hess_rows, &hc, K, nthreads);
    double dsum = 0.0;
    for (int64_t j = 0; j < K; ++j) dsum += H[j * K + j];
    double damp = 0.01 * (dsum / (double)K);
    if (damp == 0.0) damp = 1.0;
#if WQO_MUTANT != 18 /* mutant 18's mistake: the dampening is never added */
    for (int64_t j = 0; j < K; ++j) H[j * K + j] += damp;
#endif
    /* processing order: insertion sort by decreasing diagonal, stable */
    for (int64_t j = 0; j < K; ++j) perm[j] = (int32_t)j;
    if (act_order) {
        for (int64_t p = 1; p < K; ++p) {
            int32_t v = perm[p];
            int64_t q = p;
#if WQO_MUTANT == 14 /* mistake: act-order ascending */
            while (q > 0 && H[(int64_t)perm[q - 1] * K + perm[q - 1]] > H[(int64_t)v * K + v]) {
#else
            while (q > 0 && H[(int64_t)perm[q - 1] * K + perm[q - 1]] < H[(int64_t)v * K + v]) {
#endif
                perm[q] = perm[q - 1];
                --q;
            }
            perm[q] = v;
        }
    }
    for (int64_t a = 0; a < K; ++a)
        for (int64_t b = 0; b < K; ++b) Hp[a * K + b] = H[(int64_t)perm[a] * K + perm[b]];
    flags |= cholesky_lower(Hp, L, K, nthreads);
    trinv_ctx tc = {L, H, K}; /* H now holds Linv */
    run_rows(trinv_cols, &tc, K, nthreads);
    gram_ctx gc = {H, Hp, K}; /* Hp now holds H^-1 */
    run_rows(gram_rows, &gc, K, nthreads);
    flags |= cholesky_lower(Hp, L, K, nthreads);
    for (int64_t i = 0; i < K; ++i)
        for (int64_t j = 0; j < K; ++j) U[i * K + j] = L[j * K + i];
    free(H);
    free(Hp);
    free(L);
    return flags;
}

typedef struct {
    const uint16_t* W;
    int64_t K, g;
    const double* U;
    const int32_t* perm;
    const uint16_t* scales;
    const uint16_t* zeros;
    int qmin, qmax;
    int32_t* codes;
} sweep_ctx;

static void sweep_rows(void* vctx, int64_t n0, int64_t n1, uint32_t* flags) {
    sweep_ctx* c = (sweep_ctx*)vctx;
    (void)flags;
    const int64_t K = c->K, G = c->K / c->g;
    double* w = (double*)malloc(sizeof(double) * (size_t)K);
    double err[WQO_GPTQ_BLOCK];
    for (int64_t n = n0; n < n1; ++n) {
        for (int64_t p = 0; p < K; ++p) w[p] = (double)wqo_bf16_to_f32(c->W[n * K + c->perm[p]]);
        for (int64_t b0 = 0; b0 < K; b0 += WQO_GPTQ_BLOCK) {
            const int64_t b1 = b0 + WQO_GPTQ_BLOCK < K ? b0 + WQO_GPTQ_BLOCK : K;
            for (int64_t j = b0; j < b1; ++j) {
                const int64_t col = c->perm[j], gi = col / c->g;
                const uint16_t s16 = c->scales[n * G + gi];
                const int z = c->zeros ? (int)wqo_f16_to_f32(c->zeros[n * G + gi]) : 0;
                const double s = (double)wqo_f16_to_f32(s16);
                int q;
                if (isnan(w[j])) {
                    q = z;
                } else {
                    double t = rint(w[j] / s) + (double)z;
                    if (t < (double)c->qmin) t = (double)c->qmin;
                    if (t > (double)c->qmax) t = (double)c->qmax;
                    q = (int)t;
                }
                c->codes[n * K + col] = q;
                const double wh = (double)wqo_bf16_to_f32(wqo_dequant_one(s16, q, z));
#if WQO_MUTANT == 12 /* mistake: error not divided by the pivot */
                err[j - b0] = w[j] - wh;
#else
                err[j - b0] = (w[j] - wh) / c->U[j * K + j];
#endif
                for (int64_t k = j + 1; k < b1; ++k) w[k] = w[k] - err[j - b0] * c->U[j * K + k];
            }
            for (int64_t k = b1; k < K; ++k) {
                double acc = 0.0;
#if WQO_MUTANT == 13 /* mistake: tail update reads the factor transposed */
                for (int64_t j = b0; j < b1; ++j) acc = acc + err[j - b0] * c->U[k * K + j];
#else
                for (int64_t j = b0; j < b1; ++j) acc = acc + err[j - b0] * c->U[j * K + k];
#endif
                w[k] = w[k] - acc;
            }
        }
    }
    free(w);
}

/* GPTQ of W (bf16 [N][K]) with calibration X (bf16 [T][K]).  Outputs the
 * codes (original column order), the static RTN scales/zeros, the
 * processing order perm [K] and optionally U [K][K].  Returns 0, or -1 on
 * bad arguments; *flags gets WQO_FLAG_* of the RTN pass and the factor. */
int wqo_gptq(const uint16_t* W, int64_t N, int64_t K, const uint16_t* X, int64_t T, int64_t g, int symmetric,
             int act_order, int32_t* codes, uint16_t* scales, uint16_t* zeros, int32_t* perm, double* U_out,
             uint32_t* flags, int nthreads) {
    if (!W || !X || !codes || !scales || !perm || N < 1 || K < 1 || T < 1 || g < 1 || K % g != 0) return -1;
    if (!symmetric && !zeros) return -1;
    uint32_t f = 0;
    if (wqo_quantize(W, N, K, g, 4, symmetric, 0, codes, scales, symmetric ? NULL : zeros, &f, nthreads) != 0)
        return -1;
    double* U = U_out ? U_out : (double*)malloc(sizeof(double) * (size_t)(K * K));
    f |= wqo_gptq_factor(X, T, K, act_order, perm, U, nthreads);
    sweep_ctx sc = {W, K, g, U, perm, scales, symmetric ? NULL : zeros, symmetric ? -8 : 0, symmetric ? 7 : 15,
                    codes};
    run_rows(sweep_rows, &sc, N, nthreads);
    if (!U_out) free(U);
    if (flags) *flags = f;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Packing (4-bit only): 8 nibbles per uint32, low nibble first.             */
/* ------------------------------------------------------------------------ */

int wqo_pack4(const int32_t* codes, int64_t d_out, int64_t d_in, uint32_t* qweight) {
    if (!codes || !qweight || d_in % 8 != 0) return -1;
    for (int64_t r = 0; r < d_out; ++r)
        for (int64_t c8 = 0; c8 < d_in / 8; ++c8) {
            uint32_t w = 0;
            for (int j = 0; j < 8; ++j) {
                uint32_t nib = (uint32_t)codes[r * d_in + c8 * 8 + j] & 0xfu;
#if WQO_MUTANT == 7 /* mistake: high nibble first */
                w |= nib << (4 * (7 - j));
#else
                w |= nib << (4 * j);
#endif
            }
            qweight[r * (d_in / 8) + c8] = w;
        }
    return 0;
}

/* 8-bit packing (W8A16, [P1] weight-only INT8; [P2] 1.8 symmetric INT8 uses
 * [-127, 127]): 4 codes per uint32, byte j of word c holds column 4c+j as an
 * 8-bit two's complement value (bits 8j..8j+7, low byte first). */
int wqo_pack8(const int32_t* codes, int64_t d_out, int64_t d_in, uint32_t* qweight) {
    if (!codes || !qweight || d_in % 4 != 0) return -1;
    for (int64_t r = 0; r < d_out; ++r)
        for (int64_t c4 = 0; c4 < d_in / 4; ++c4) {
            uint32_t w = 0;
            for (int j = 0; j < 4; ++j)
#if WQO_MUTANT == 8 /* mistake: high byte first */
                w |= ((uint32_t)codes[r * d_in + c4 * 4 + j] & 0xffu) << (8 * (3 - j));
#else
                w |= ((uint32_t)codes[r * d_in + c4 * 4 + j] & 0xffu) << (8 * j);
#endif
            qweight[r * (d_in / 4) + c4] = w;
        }
    return 0;
}

int wqo_unpack8(const uint32_t* qweight, int64_t d_out, int64_t d_in, int32_t* codes) {
    if (!codes || !qweight || d_in % 4 != 0) return -1;
    for (int64_t r = 0; r < d_out; ++r)
        for (int64_t c = 0; c < d_in; ++c) {
            int32_t b = (int32_t)((qweight[r * (d_in / 4) + c / 4] >> (8 * (c % 4))) & 0xffu);
            codes[r * d_in + c] = b >= 128 ? b - 256 : b;
        }
    return 0;
}

/* Inverse of wqo_pack4: symmetric nibbles are read as 4-bit two's complement. */
int wqo_unpack4(const uint32_t* qweight, int64_t d_out, int64_t d_in, int symmetric,
                int32_t* codes) {
    if (!codes || !qweight || d_in % 8 != 0) return -1;
    for (int64_t r = 0; r < d_out; ++r)
        for (int64_t c = 0; c < d_in; ++c) {
            uint32_t w = qweight[r * (d_in / 8) + c / 8];
            int32_t nib = (int32_t)((w >> (4 * (c % 8))) & 0xfu);
#if WQO_MUTANT != 16 /* mutant 16's mistake: symmetric nibbles read without sign extension */
            if (symmetric && nib >= 8) nib -= 16;
#endif
            codes[r * d_in + c] = nib;
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Dequantize: x_hat = s (q - z), rounded once to bf16 [P1 Affine].          */
/* ------------------------------------------------------------------------ */

/* The product of an fp16 scale (11 significant bits) and an integer of at
 * most 8 bits (|q - z| <= 255) has at most 19 significant bits and lies in
 * the binary32 range, so it is exact in double and in float; the only
 * rounding is the final one to bf16. */
uint16_t wqo_dequant_one(uint16_t s16, int32_t q, int32_t z) {
#if WQO_MUTANT == 6 /* mistake: zero point dropped */
    z = 0;
#endif
    double prod = (double)wqo_f16_to_f32(s16) * (double)(q - z);
    float pf = (float)prod; /* exact, see above */
#if WQO_MUTANT == 24 /* mistake: truncated to bf16 instead of rounded to nearest even */
    uint32_t bits;
    memcpy(&bits, &pf, 4);
    return (uint16_t)(bits >> 16);
#else
    return wqo_f32_to_bf16(pf);
#endif
}

typedef struct {
    const int32_t* codes;
    const uint16_t* scales;
    const uint16_t* zeros;
    int64_t d_in, g;
    uint16_t* W_hat;
} deq_ctx;

static void deq_rows(void* vctx, int64_t r0, int64_t r1, uint32_t* flags) {
    (void)flags;
    deq_ctx* c = (deq_ctx*)vctx;
    int64_t ng = c->d_in / c->g;
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t k = 0; k < c->d_in; ++k) {
            int64_t gi = r * ng + k / c->g;
            int32_t z = c->zeros ? (int32_t)wqo_f16_to_f32(c->zeros[gi]) : 0;
            c->W_hat[r * c->d_in + k] = wqo_dequant_one(c->scales[gi], c->codes[r * c->d_in + k], z);
        }
}

/* codes int32 [d_out][d_in]; scales/zeros fp16 bits [d_out][d_in/g]
 * (zeros NULL = symmetric); W_hat bf16 bits [d_out][d_in]. */
int wqo_dequantize(const int32_t* codes, const uint16_t* scales, const uint16_t* zeros,
                   int64_t d_out, int64_t d_in, int64_t g, uint16_t* W_hat, int nthreads) {
    if (!codes || !scales || !W_hat || g <= 0 || d_in % g != 0) return -1;
    deq_ctx c = {codes, scales, zeros, d_in, g, W_hat};
    run_rows(deq_rows, &c, d_out, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Linear: y[m,n] = sum_k W_hat[n,k] x[m,k] in fp64, plus the error scale    */
/* A[m,n] = sum_k |W_hat[n,k] x[m,k]|.                                        */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t* X;
    int64_t M;
    const uint16_t* W_hat;
    int64_t K;
    double* Y;
    double* A;
    int64_t N;
} lin_ctx;

static void lin_rows(void* vctx, int64_t n0, int64_t n1, uint32_t* flags) {
    (void)flags;
    lin_ctx* c = (lin_ctx*)vctx;
    for (int64_t n = n0; n < n1; ++n)
        for (int64_t m = 0; m < c->M; ++m) {
            double acc = 0.0, aacc = 0.0;
#if WQO_MUTANT == 22 /* mistake: the last input channel is dropped */
            for (int64_t k = 0; k < c->K - 1; ++k) {
#else
            for (int64_t k = 0; k < c->K; ++k) {
#endif
#if WQO_MUTANT == 5 /* mistake: transposed weight operand */
                double t = (double)wqo_bf16_to_f32(c->W_hat[(k % c->N) * c->K + (n % c->K)]) *
                           (double)wqo_bf16_to_f32(c->X[m * c->K + k]);
#else
                double t = (double)wqo_bf16_to_f32(c->W_hat[n * c->K + k]) *
                           (double)wqo_bf16_to_f32(c->X[m * c->K + k]);
#endif
                acc += t;
#if WQO_MUTANT == 23 /* mistake: the error scale sums signed terms */
                aacc += t;
#else
                aacc += fabs(t);
#endif
            }
            c->Y[m * c->N + n] = acc;
            if (c->A) c->A[m * c->N + n] = aacc;
        }
}

/* X bf16 bits [M][K]; W_hat bf16 bits [N][K]; Y, A fp64 [M][N] (A may be
 * NULL).  Rows of W_hat are split across threads. */
int wqo_linear(const uint16_t* X, int64_t M, const uint16_t* W_hat, int64_t N, int64_t K,
               double* Y, double* A, int nthreads) {
    if (!X || !W_hat || !Y || M < 0 || N < 0 || K < 0) return -1;
    lin_ctx c = {X, M, W_hat, K, Y, A, N};
    run_rows(lin_rows, &c, N, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Artifact bytes [P1 Memory arithmetic, Group scale overhead]:              */
/*   payload = P * b / 8; one fp16 scale per group of g; one fp16 zero per   */
/*   group when asymmetric.                                                  */
/* ------------------------------------------------------------------------ */

int wqo_artifact_bytes(int64_t params, int bits, int64_t g, int symmetric, double* payload,
                       double* scale_bytes, double* zero_bytes) {
    if (g <= 0 || bits <= 0) return -1;
    *payload = (double)params * (double)bits / 8.0;
    *scale_bytes = 2.0 * (double)params / (double)g;
    *zero_bytes = symmetric ? 0.0 : 2.0 * (double)params / (double)g;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Array forms of the conversions (used by the pins to compare whole ranges  */
/* of inputs against independent library conversions).                      */
/* ------------------------------------------------------------------------ */

void wqo_f32_to_f16_array(const float* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = wqo_f32_to_f16(x[i]);
}

void wqo_f32_to_bf16_array(const float* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = wqo_f32_to_bf16(x[i]);
}

void wqo_f16_to_f32_array(const uint16_t* h, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = wqo_f16_to_f32(h[i]);
}
