/*
 * qz_oracle.c -- plain, slow, scalar CPU oracle for group-wise affine weight
 * quantization and the weight-only dequantize-matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA library; the two meet only through the seeded input generator.
 *
 * Sources (the HF Transformers "Quantization concepts" guide, section
 * "Mapping values to fewer bits"; the taqaniya.com "What is quantization"
 * page, IBM absmax example; the GPTQ explainer at azimuth.plus):
 *   scale        S = (val_max - val_min) / (q_max - q_min)
 *   zero-point   Z = q_min - round(val_min / S)
 *   quantize     q = round(x / S + Z)
 *   dequantize   x ~ S * (q - Z)
 *   symmetric    range [-a, a], Z fixed at 0, only S stored (int8: +-127)
 *   granularity  per-tensor / per-channel (one per output row) / per-group of
 *                consecutive values along a row (section "Choose granularity")
 *   int4 packing two codes per byte, first in the low nibble (section
 *                "int8 and int4", packing figure)
 *
 * Readings where the pages are silent (each is listed with its reason in the
 * design notes of the repository):
 *   - round() is round-half-to-even (rintf in the default rounding mode);
 *   - q is clamped to [q_min, q_max];
 *   - the asymmetric range is extended to contain 0.0, since Z is defined as
 *     the integer that represents 0.0;
 *   - S is computed in IEEE fp32 and stored as bf16 rounded toward +inf, and
 *     quantization divides by that stored value (so every x/S+Z stays inside
 *     [q_min - 1/2, q_max + 1/2]);
 *   - S == 0 (an all-zero group) is replaced by 1.0;
 *   - int4 asymmetric codes are unsigned [0, 15]; int4 symmetric codes are
 *     [-7, 7]; int8 asymmetric codes are [-128, 127]; int8 symmetric [-127, 127];
 *   - the dequantized weight is bf16, rounded to nearest-even from the exact
 *     fp32 product S*(q - Z);
 *   - the matmul reference is an fp64 dot product over those bf16 weights.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -fPIC -shared
 * (no FMA contraction, no fast-math, no flush-to-zero).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* bf16 <-> fp32 bit conversions                                        */
/* ------------------------------------------------------------------ */

static float f32_of_bits(uint32_t b) { float f; memcpy(&f, &b, sizeof f); return f; }
static uint32_t bits_of_f32(float f) { uint32_t b; memcpy(&b, &f, sizeof b); return b; }

/* A bf16 value is the upper 16 bits of an fp32: widening is exact. */
float qzo_bf16_to_f32(uint16_t h) { return f32_of_bits((uint32_t)h << 16); }

/* fp32 -> bf16, round to nearest, ties to even (finite inputs; NaN kept quiet). */
uint16_t qzo_f32_to_bf16_rne(float x)
{
    uint32_t b = bits_of_f32(x);
    if ((b & 0x7F800000u) == 0x7F800000u && (b & 0x007FFFFFu) != 0)
        return (uint16_t)((b >> 16) | 0x0040u);
    uint32_t kept = b & 0xFFFF0000u;      /* truncated magnitude (sign-magnitude) */
    uint32_t dropped = b & 0x0000FFFFu;   /* the 16 bits that do not fit */
    int kept_is_odd = (kept >> 16) & 1u;
    if (dropped > 0x8000u || (dropped == 0x8000u && kept_is_odd))
        kept += 0x00010000u;              /* one bf16 ulp away from zero */
    return (uint16_t)(kept >> 16);
}

/* fp32 -> bf16 rounded toward +infinity, for the non-negative scale S. */
uint16_t qzo_f32_to_bf16_up(float s)
{
    uint32_t b = bits_of_f32(s);
    uint32_t kept = b & 0xFFFF0000u;
    if (b & 0x0000FFFFu)
        kept += 0x00010000u;              /* next bf16 above (s > 0) */
    return (uint16_t)(kept >> 16);
}

/* ------------------------------------------------------------------ */
/* Code ranges (quantization concepts guide: int8 is [-128, 127], int4   */
/* holds 16 integers; IBM example: symmetric int8 range is -127..127).   */
/* ------------------------------------------------------------------ */

int qzo_code_range(int bits, int symmetric, int *qmin, int *qmax)
{
    if (bits != 4 && bits != 8) return -1;
    if (symmetric) {
        *qmax = (1 << (bits - 1)) - 1;   /* 7 or 127 */
        *qmin = -*qmax;
    } else if (bits == 4) {
        *qmin = 0;                       /* unsigned nibble */
        *qmax = 15;
    } else {
        *qmin = -128;
        *qmax = 127;
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* One group: scale, zero-point, codes.                                  */
/* x[0..n) are consecutive values of one group (fp32, exact bf16 values). */
/* ------------------------------------------------------------------ */

/* Scale and zero-point of one group from its values x[0..n) (fp32). */
static void group_scale_zero(const float *x, int64_t n, int bits, int symmetric,
                             uint16_t *scale_bf16, int32_t *zero)
{
    int qmin, qmax;
    qzo_code_range(bits, symmetric, &qmin, &qmax);

    float S;
    float vmin = 0.0f, vmax = 0.0f;       /* the range always contains 0.0 */
    if (symmetric) {
        float a = 0.0f;                   /* a = max |x| */
        for (int64_t i = 0; i < n; ++i) {
            float m = fabsf(x[i]);
            if (m > a) a = m;
        }
        S = a / (float)qmax;              /* range [-a, a] onto [-qmax, qmax] */
    } else {
        for (int64_t i = 0; i < n; ++i) {
            if (x[i] < vmin) vmin = x[i];
            if (x[i] > vmax) vmax = x[i];
        }
        S = (vmax - vmin) / (float)(qmax - qmin);
    }
    if (S == 0.0f) S = 1.0f;              /* all-zero group */

    uint16_t Sb = qzo_f32_to_bf16_up(S);  /* stored scale */
    float Sf = qzo_bf16_to_f32(Sb);       /* the value every later step uses */

    int32_t Z = 0;
    if (!symmetric)
        Z = qmin - (int32_t)rintf(vmin / Sf);
    *scale_bf16 = Sb;
    *zero = Z;
}

/* Code of one value x (fp32) under the stored scale and zero-point. */
static int32_t code_of(float x, uint16_t scale_bf16, int32_t Z, int qmin, int qmax)
{
    float Sf = qzo_bf16_to_f32(scale_bf16);
    float u = x / Sf + (float)Z;          /* divide, then shift by Z, in fp32 */
    float r = rintf(u);                   /* round half to even */
    int32_t c = (int32_t)r;
    if (c < qmin) c = qmin;
    if (c > qmax) c = qmax;
    return c;
}

static void quantize_group(const float *x, int64_t n, int bits, int symmetric,
                           uint16_t *scale_bf16, int32_t *zero, int32_t *q)
{
    int qmin, qmax;
    qzo_code_range(bits, symmetric, &qmin, &qmax);
    group_scale_zero(x, n, bits, symmetric, scale_bf16, zero);
    for (int64_t i = 0; i < n; ++i)
        q[i] = code_of(x[i], *scale_bf16, *zero, qmin, qmax);
}

/* ------------------------------------------------------------------ */
/* Tensor layout                                                         */
/*   w      : N x K row-major values (fp32 carrying bf16 values)         */
/*   groups : group_size g > 0 with K % g == 0 -> groups of g consecutive */
/*            values along each row, scales[n*(K/g) + k/g];              */
/*            g == K is per-channel; g == 0 is per-tensor (one group).   */
/*   codes  : bits 4 -> N x K/2 bytes, value k in the low nibble when k   */
/*            is even, in the high nibble when k is odd;                  */
/*            bits 8 -> N x K bytes (two's complement).                   */
/*   zeros  : one byte per group (asymmetric only): unsigned for int4,    */
/*            two's complement for int8.                                  */
/* ------------------------------------------------------------------ */

static int check_shape(int64_t N, int64_t K, int bits, int64_t g)
{
    if (N < 1 || K < 1) return -1;
    if (g < 0) return -1;
    if (g > 0 && (K % g) != 0) return -1;
    if (bits == 4 && (K % 2) != 0) return -1;
    return 0;
}

static void store_code(uint8_t *codes, int64_t N, int64_t K, int bits,
                       int64_t n, int64_t k, int32_t c)
{
    (void)N;
    if (bits == 8) {
        codes[n * K + k] = (uint8_t)(int8_t)c;
    } else {
        uint8_t nib = (uint8_t)(c & 0xF);
        uint8_t *byte = &codes[n * (K / 2) + k / 2];
        if ((k & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | nib);
        else              *byte = (uint8_t)((*byte & 0x0F) | (nib << 4));
    }
}

static int32_t load_code(const uint8_t *codes, int64_t K, int bits, int symmetric,
                         int64_t n, int64_t k)
{
    if (bits == 8)
        return (int32_t)(int8_t)codes[n * K + k];
    uint8_t byte = codes[n * (K / 2) + k / 2];
    int32_t nib = (k & 1) ? (byte >> 4) : (byte & 0xF);
    if (symmetric && nib >= 8) nib -= 16;   /* two's complement nibble */
    return nib;
}

/* Quantize and pack.  Returns 0 on success, -1 on a bad argument. */
int qzo_quantize_pack(const float *w, int64_t N, int64_t K, int bits, int symmetric,
                      int64_t g, uint8_t *codes, uint16_t *scales, uint8_t *zeros)
{
    int qmin, qmax;
    if (qzo_code_range(bits, symmetric, &qmin, &qmax) || check_shape(N, K, bits, g))
        return -1;

    if (g == 0) {
        /* per-tensor: one group spanning the whole matrix */
        int64_t total = N * K;
        int32_t *q = (int32_t *)malloc((size_t)total * sizeof(int32_t));
        if (!q) return -1;
        uint16_t Sb; int32_t Z;
        quantize_group(w, total, bits, symmetric, &Sb, &Z, q);
        for (int64_t n = 0; n < N; ++n)
            for (int64_t k = 0; k < K; ++k)
                store_code(codes, N, K, bits, n, k, q[n * K + k]);
        scales[0] = Sb;
        if (!symmetric) zeros[0] = (uint8_t)(int8_t)Z;
        free(q);
        return 0;
    }

    int64_t gpr = K / g;   /* groups per row */
    int failed = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n) {
        int32_t *q = (int32_t *)malloc((size_t)g * sizeof(int32_t));
        if (!q) { failed = 1; continue; }
        for (int64_t j = 0; j < gpr; ++j) {
            uint16_t Sb; int32_t Z;
            quantize_group(&w[n * K + j * g], g, bits, symmetric, &Sb, &Z, q);
            for (int64_t i = 0; i < g; ++i)
                store_code(codes, N, K, bits, n, j * g + i, q[i]);
            scales[n * gpr + j] = Sb;
            if (!symmetric) zeros[n * gpr + j] = (uint8_t)(int8_t)Z;
        }
        free(q);
    }
    return failed ? -1 : 0;
}

/* Dequantize: w_hat = bf16_rne( S * (q - Z) ).  The fp32 product of an
 * 8-bit-significand scale and an integer of at most 8 bits is exact, so the
 * only rounding is the final one to bf16. */
int qzo_dequantize(const uint8_t *codes, const uint16_t *scales, const uint8_t *zeros,
                   int64_t N, int64_t K, int bits, int symmetric, int64_t g,
                   uint16_t *w_hat)
{
    int qmin, qmax;
    if (qzo_code_range(bits, symmetric, &qmin, &qmax) || check_shape(N, K, bits, g))
        return -1;
    int64_t gpr = (g == 0) ? 0 : K / g;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int64_t gi = (g == 0) ? 0 : n * gpr + k / g;
            float Sf = qzo_bf16_to_f32(scales[gi]);
            int32_t Z = 0;
            if (!symmetric) {
                Z = (bits == 4) ? (int32_t)zeros[gi] : (int32_t)(int8_t)zeros[gi];
            }
            int32_t q = load_code(codes, K, bits, symmetric, n, k);
            float prod = Sf * (float)(q - Z);
            w_hat[n * K + k] = qzo_f32_to_bf16_rne(prod);
        }
    }
    return 0;
}

/* Reference matmul in fp64 over bf16 operands:
 *   y[m][n]     = sum_k a[m][k] * w_hat[n][k]
 *   abs_y[m][n] = sum_k |a[m][k] * w_hat[n][k]|   (for the tolerance bound)
 * a is M x K, w_hat is N x K (both bf16 bits, row-major). */
int qzo_matmul_f64(const uint16_t *a, const uint16_t *w_hat, int64_t M, int64_t N,
                   int64_t K, double *y, double *abs_y)
{
    if (M < 0 || N < 0 || K < 0) return -1;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            double s = 0.0, sa = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = (double)qzo_bf16_to_f32(a[m * K + k]) *
                           (double)qzo_bf16_to_f32(w_hat[n * K + k]);
                s += p;
                sa += fabs(p);
            }
            y[m * N + n] = s;
            if (abs_y) abs_y[m * N + n] = sa;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* FP4 with block scales (quantization concepts guide, section "FP4 with */
/* block scales"; the FP8 section for E4M3).                              */
/*   E2M1: 1 sign, 2 exponent, 1 mantissa bit; the magnitudes 0, 0.5, 1,  */
/*   1.5, 2, 3, 4, 6 (codes 0..7 in that order, sign in bit 3).           */
/*   MXFP4: a power-of-two scale per block (only the exponent shifts).    */
/*   NVFP4: smaller blocks with an FP8 (E4M3) scale, plus one scale for   */
/*   the tensor that keeps the block scales in range.                     */
/* Readings (the page gives no block sizes and no rule for choosing a     */
/* scale):                                                                */
/*   - MXFP4 blocks are 32 values, NVFP4 blocks 16 (NVFP4's are the       */
/*     smaller), consecutive along a row;                                 */
/*   - MXFP4 scale: 2^e with e the smallest integer such that             */
/*     max|x| / 2^e <= 6 (no value saturates), clamped to [-127, 127],    */
/*     stored as the E8M0 byte e + 127; an all-zero block has e = -127;   */
/*   - NVFP4 tensor scale: s_t = fp32(amax / 2688) (2688 = 6 x 448, the    */
/*     largest E2M1 value times the largest E4M3 value), 1 for an all-    */
/*     zero tensor; block scale: the smallest E4M3 value >= fp32(amax_b / */
/*     fp32(6 s_t)) (rounded up, like the bf16 scales of the integer      */
/*     formats), at most 448, 0 for an all-zero block;                    */
/*   - element codes: x divided by the block's effective scale (2^e, or    */
/*     fp32(E4M3(s_b) x s_t)) in fp32, then rounded to the nearest E2M1   */
/*     magnitude, ties to the even mantissa bit, saturating at 6;          */
/*   - dequantized weight (bf16 output): MXFP4 e2m1 x 2^e; NVFP4           */
/*     bf16_rne(fp32(fp32(e2m1 x E4M3(s_b)) x s_t)) (the inner product is  */
/*     exact);                                                            */
/*   - the matmul reference uses the exact product e2m1 x scale(s) in fp64.*/
/* ------------------------------------------------------------------ */

static const double e2m1_mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Nearest E2M1 code (sign in bit 3) of v, ties to the even mantissa bit
 * (codes with an even index), saturating at 6. */
static uint8_t e2m1_code(float v)
{
    double a = fabs((double)v);
    int best = 0;
    for (int i = 1; i < 8; ++i) {
        double di = fabs(a - e2m1_mag[i]), db = fabs(a - e2m1_mag[best]);
        if (di < db || (di == db && (i % 2) == 0 && (best % 2) == 1)) best = i;
    }
    if (a > 6.0) best = 7;
    uint8_t code = (uint8_t)best;
    if (v < 0.0f && best != 0) code |= 0x8;
    return code;
}

/* E4M3 (FP8, 4 exponent bits with bias 7, 3 mantissa bits, finite max 448)
 * byte -> value. */
double qzo_e4m3_to_f64(uint8_t b)
{
    int s = (b >> 7) & 1, e = (b >> 3) & 0xF, m = b & 7;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* The smallest non-negative E4M3 value >= t (t >= 0), capped at 448. */
static uint8_t e4m3_round_up(float t)
{
    if (!(t > 0.0f)) return 0;
    for (int b = 1; b <= 0x7E; ++b)               /* 0x7E = 448, 0x7F is NaN */
        if (qzo_e4m3_to_f64((uint8_t)b) >= (double)t) return (uint8_t)b;
    return 0x7E;
}

double qzo_e2m1_to_f64(uint8_t code)
{
    double v = e2m1_mag[code & 7];
    return (code & 8) ? -v : v;
}

/* kind 0 = MXFP4 (block 32, E8M0), 1 = NVFP4 (block 16, E4M3 + tensor scale). */
static int fp4_block(int kind) { return kind == 0 ? 32 : 16; }

int qzo_fp4_quantize(const float *w, int64_t N, int64_t K, int kind, uint8_t *codes,
                     uint8_t *block_scales, float *tensor_scale)
{
    if ((kind != 0 && kind != 1) || N < 1 || K < 1) return -1;
    const int bs = fp4_block(kind);
    if (K % bs != 0) return -1;
    float s_t = 1.0f;
    if (kind == 1) {
        float amax = 0.0f;
        for (int64_t i = 0; i < N * K; ++i)
            if (fabsf(w[i]) > amax) amax = fabsf(w[i]);
        s_t = amax > 0.0f ? amax / 2688.0f : 1.0f;
        *tensor_scale = s_t;
    }
    const int64_t bpr = K / bs;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < bpr; ++b) {
            const float *x = &w[n * K + b * bs];
            float amax = 0.0f;
            for (int i = 0; i < bs; ++i)
                if (fabsf(x[i]) > amax) amax = fabsf(x[i]);
            float scale;
            uint8_t sb;
            if (kind == 0) {
                int e = -127;
                if (amax > 0.0f) {
                    e = (int)floor(log2((double)amax / 6.0)) - 1;
                    while ((double)amax > 6.0 * ldexp(1.0, e)) ++e;   /* smallest e */
                    if (e < -127) e = -127;
                    if (e > 127) e = 127;
                }
                sb = (uint8_t)(e + 127);
                scale = (float)ldexp(1.0, e);
            } else {
                float t = amax / (6.0f * s_t);
                sb = e4m3_round_up(t);
                scale = (float)qzo_e4m3_to_f64(sb) * s_t;
            }
            block_scales[n * bpr + b] = sb;
            for (int i = 0; i < bs; ++i) {
                const int64_t k = b * bs + i;
                uint8_t c = scale > 0.0f ? e2m1_code(x[i] / scale) : 0;
                uint8_t *byte = &codes[n * (K / 2) + k / 2];
                if ((k & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | c);
                else              *byte = (uint8_t)((*byte & 0x0F) | (c << 4));
            }
        }
    }
    return 0;
}

/* Exact dequantized value (fp64) of element (n, k), and its bf16 output. */
static double fp4_value(const uint8_t *codes, const uint8_t *block_scales, float s_t,
                        int64_t K, int kind, int64_t n, int64_t k)
{
    const int bs = fp4_block(kind);
    uint8_t byte = codes[n * (K / 2) + k / 2];
    uint8_t c = (k & 1) ? (byte >> 4) : (byte & 0xF);
    uint8_t sb = block_scales[n * (K / bs) + k / bs];
    double q = qzo_e2m1_to_f64(c);
    if (kind == 0) return q * ldexp(1.0, (int)sb - 127);
    return q * qzo_e4m3_to_f64(sb) * (double)s_t;
}

int qzo_fp4_dequantize(const uint8_t *codes, const uint8_t *block_scales, const float *tensor_scale,
                       int64_t N, int64_t K, int kind, uint16_t *w_hat, double *w_exact)
{
    if ((kind != 0 && kind != 1) || N < 1 || K < 1 || K % fp4_block(kind) != 0) return -1;
    const float s_t = kind == 1 ? *tensor_scale : 1.0f;
    const int bs = fp4_block(kind);
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            if (w_exact) w_exact[n * K + k] = fp4_value(codes, block_scales, s_t, K, kind, n, k);
            if (w_hat) {
                uint8_t byte = codes[n * (K / 2) + k / 2];
                uint8_t c = (k & 1) ? (byte >> 4) : (byte & 0xF);
                uint8_t sb = block_scales[n * (K / bs) + k / bs];
                float v;
                if (kind == 0) {
                    v = (float)(qzo_e2m1_to_f64(c) * ldexp(1.0, (int)sb - 127));
                } else {
                    float p = (float)qzo_e2m1_to_f64(c) * (float)qzo_e4m3_to_f64(sb);  /* exact */
                    v = p * s_t;
                }
                w_hat[n * K + k] = qzo_f32_to_bf16_rne(v);
            }
        }
    return 0;
}

/* fp64 reference matmul over exact dequantized weights (N x K fp64):
 * y[m][n] = sum_k a[m][k] w[n][k] and sum_k |a w|. */
int qzo_matmul_f64_exact(const uint16_t *a, const double *w, int64_t M, int64_t N, int64_t K,
                         double *y, double *abs_y)
{
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0, acc_abs = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = (double)qzo_bf16_to_f32(a[m * K + k]) * w[n * K + k];
                acc += p;
                acc_abs += fabs(p);
            }
            y[m * N + n] = acc;
            abs_y[m * N + n] = acc_abs;
        }
    return 0;
}

/* y = a @ w^T and sum_k |a w| in fp64 for fp64 a (M x K) and w (N x K):
 * the W4A4 reference, both operands already exact dequantized FP4 values
 * (Quantization concepts guide, "Quantize weights or activations": NVFP4
 * W4A4 quantizes the activations as well as the weights). */
int qzo_matmul_f64_ab(const double *a, const double *w, int64_t M, int64_t N, int64_t K,
                      double *y, double *abs_y)
{
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m < M; ++m) {
            double sum = 0.0, sum_abs = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double t = a[m * K + k] * w[n * K + k];
                sum += t;
                sum_abs += fabs(t);
            }
            y[m * N + n] = sum;
            abs_y[m * N + n] = sum_abs;
        }
    return 0;
}

/* ------------------------------------------------------------------ */
/* GPTQ layer-wise quantizer (GPTQ explainer, azimuth.plus/paper/gptq).  */
/*                                                                        */
/* The page's steps, in its order:                                        */
/*   - input: the layer's weights W (rows = outputs, columns = inputs)    */
/*     and H = 2 X X^T from calibration data X (one column per sample);   */
/*   - a small damping term lambda I is added to H;                       */
/*   - OBQ: quantize the weights one at a time and, after each, adjust    */
/*     every weight not yet quantized to compensate the rounding error    */
/*     w_q - quant(w_q), in the direction given by the inverse Hessian;   */
/*   - first innovation: one fixed column order for every row, so the     */
/*     inverse Hessian is shared by all rows;                             */
/*   - second innovation: lazy batches of B = 128 columns -- the updates  */
/*     inside a block are applied at once, the rest of the matrix gets    */
/*     one large update when the block is done;                           */
/*   - third innovation: the Cholesky decomposition of H^-1 is computed   */
/*     once, and the entries the updates need are read from it row by     */
/*     row.                                                               */
/* The display formulas were lost in the page's extraction; this restates */
/* the standard forms the prose describes.  With U the upper Cholesky     */
/* factor of H^-1 (H^-1 = U^T U), the row of U at column j, scaled by     */
/* 1 / U[j][j], is the OBQ update direction of the not-yet-quantized      */
/* columns after columns 0..j-1 were eliminated, so quantizing column j   */
/* is: e = (w_j - quant(w_j)) / U[j][j]; w_k -= e * U[j][k] for k > j.    */
/*                                                                        */
/* Readings where the page is silent (listed in the design notes):        */
/*   - lambda = damp * mean(diag H) (damp = 0.01 by default), or 1 when   */
/*     that mean is 0;                                                    */
/*   - quant() is this file's round-to-nearest quantizer: a group's       */
/*     scale and zero-point come from the group's weights as they stand   */
/*     (already compensated) when its first column is reached, and every  */
/*     column is coded from its own compensated value; both use the fp32  */
/*     arithmetic of quantize_pack on the fp64 weights rounded to fp32;   */
/*   - every other step is fp64; group starts and block starts must nest  */
/*     (g % B == 0 or B % g == 0), so a group's weights are up to date    */
/*     when its scale is taken.                                           */
/* ------------------------------------------------------------------ */

/* In-place Cholesky A = L L^T of an n x n symmetric positive definite
 * matrix (row-major fp64); on return the lower triangle holds L and the
 * strict upper triangle is zero.  Returns -1 if A is not positive definite.
 * (Rows below the pivot are independent: OpenMP over them.) */
static int cholesky_lower(double *A, int64_t n)
{
    for (int64_t j = 0; j < n; ++j) {
        double d = A[j * n + j];
        for (int64_t k = 0; k < j; ++k) d -= A[j * n + k] * A[j * n + k];
        if (!(d > 0.0)) return -1;
        double ljj = sqrt(d);
        A[j * n + j] = ljj;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
        for (int64_t i = j + 1; i < n; ++i) {
            double v = A[i * n + j];
            for (int64_t k = 0; k < j; ++k) v -= A[i * n + k] * A[j * n + k];
            A[i * n + j] = v / ljj;
        }
        for (int64_t i = 0; i < j; ++i) A[i * n + j] = 0.0;
    }
    return 0;
}

/* Inverse of an SPD matrix from its Cholesky factor: A^-1 = L^-T L^-1.
 * L^-1 by forward substitution, one column c at a time (stored transposed:
 * LiT[c][i] = (L^-1)[i][c], so the sums run over contiguous memory), then
 * the product (A^-1)[i][j] = sum_k (L^-1)[k][i] (L^-1)[k][j]. */
static void spd_inverse_from_cholesky(const double *L, double *Ainv, int64_t n)
{
    double *LiT = (double *)calloc((size_t)(n * n), sizeof(double));
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 8)
#endif
    for (int64_t c = 0; c < n; ++c) {             /* column c of L^-1 */
        double *col = &LiT[c * n];
        for (int64_t i = c; i < n; ++i) {
            double v = (i == c) ? 1.0 : 0.0;
            for (int64_t k = c; k < i; ++k) v -= L[i * n + k] * col[k];
            col[i] = v / L[i * n + i];
        }
    }
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 8)
#endif
    for (int64_t i = 0; i < n; ++i)
        for (int64_t j = 0; j < n; ++j) {
            double v = 0.0;
            int64_t k0 = i > j ? i : j;
            for (int64_t k = k0; k < n; ++k) v += LiT[i * n + k] * LiT[j * n + k];
            Ainv[i * n + j] = v;
        }
    free(LiT);
}

/* Upper Cholesky factor: A = U^T U (U upper, positive diagonal).  Built in
 * the transposed array UT[j][i] = U[i][j] so the sums are contiguous. */
static int cholesky_upper(const double *A, double *U, int64_t n)
{
    double *UT = (double *)calloc((size_t)(n * n), sizeof(double));
    if (!UT) return -1;
    int rc = 0;
    for (int64_t i = 0; i < n && rc == 0; ++i) {
        double d = A[i * n + i];
        for (int64_t k = 0; k < i; ++k) d -= UT[i * n + k] * UT[i * n + k];
        if (!(d > 0.0)) { rc = -1; break; }
        double uii = sqrt(d);
        UT[i * n + i] = uii;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
        for (int64_t j = i + 1; j < n; ++j) {
            double v = A[i * n + j];
            for (int64_t k = 0; k < i; ++k) v -= UT[i * n + k] * UT[j * n + k];
            UT[j * n + i] = v / uii;
        }
    }
    for (int64_t i = 0; i < n; ++i)
        for (int64_t j = 0; j < n; ++j) U[i * n + j] = j >= i ? UT[j * n + i] : 0.0;
    free(UT);
    return rc;
}

/* The damped Hessian H = 2 X X^T + lambda I and the upper Cholesky factor U
 * of its inverse.  x is n_samples x K (one calibration sample per row, bf16
 * bits), so X = x^T.  Returns -1 if the damped Hessian is not positive
 * definite. */
int qzo_gptq_hessian_factor(const uint16_t *x, int64_t K, int64_t n_samples, double damp,
                            double *H, double *U)
{
    if (K < 1 || n_samples < 0 || !(damp >= 0.0)) return -1;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t a = 0; a < K; ++a)
        for (int64_t b = 0; b < K; ++b) {
            double v = 0.0;
            for (int64_t t = 0; t < n_samples; ++t)
                v += (double)qzo_bf16_to_f32(x[t * K + a]) * (double)qzo_bf16_to_f32(x[t * K + b]);
            H[a * K + b] = 2.0 * v;
        }
    double mean = 0.0;
    for (int64_t a = 0; a < K; ++a) mean += H[a * K + a];
    mean /= (double)K;
    double lambda = mean > 0.0 ? damp * mean : 1.0;
    for (int64_t a = 0; a < K; ++a) H[a * K + a] += lambda;

    double *L = (double *)malloc((size_t)(K * K) * sizeof(double));
    double *Hinv = (double *)malloc((size_t)(K * K) * sizeof(double));
    int rc = -1;
    if (L && Hinv) {
        memcpy(L, H, (size_t)(K * K) * sizeof(double));
        if (cholesky_lower(L, K) == 0) {
            spd_inverse_from_cholesky(L, Hinv, K);
            rc = cholesky_upper(Hinv, U, K);
        }
    }
    free(L);
    free(Hinv);
    return rc;
}

/* GPTQ over the N x K weights w (fp32 values) given U (the upper Cholesky
 * factor of the damped inverse Hessian, K x K fp64), in lazy blocks of
 * `block` columns; writes the packed codes, scales and zeros of the format
 * (group_size g > 0) and the final compensated weights w_out (N x K fp64,
 * may be NULL).  Returns -1 on a bad argument. */
int qzo_gptq_quantize_with_factor(const float *w, const double *U, int64_t N, int64_t K,
                                  int64_t block, int bits, int symmetric, int64_t g,
                                  uint8_t *codes, uint16_t *scales, uint8_t *zeros,
                                  double *w_out)
{
    int qmin, qmax;
    if (qzo_code_range(bits, symmetric, &qmin, &qmax) || check_shape(N, K, bits, g)) return -1;
    if (g == 0 || block < 1 || (g % block != 0 && block % g != 0)) return -1;
    int64_t gpr = K / g;
    int failed = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t n = 0; n < N; ++n) {             /* rows are independent */
        double *W = (double *)malloc((size_t)K * sizeof(double));
        double *E = (double *)malloc((size_t)block * sizeof(double));
        float *grp = (float *)malloc((size_t)g * sizeof(float));
        if (!W || !E || !grp) { failed = 1; free(W); free(E); free(grp); continue; }
        for (int64_t k = 0; k < K; ++k) W[k] = (double)w[n * K + k];
        uint16_t Sb = 0;
        int32_t Z = 0;
        for (int64_t i = 0; i < K; i += block) {
            int64_t end = i + block < K ? i + block : K;
            for (int64_t j = i; j < end; ++j) {
                if (j % g == 0) {                 /* a group starts: its scale and zero */
                    for (int64_t k = 0; k < g; ++k) grp[k] = (float)W[j + k];
                    group_scale_zero(grp, g, bits, symmetric, &Sb, &Z);
                    scales[n * gpr + j / g] = Sb;
                    if (!symmetric) zeros[n * gpr + j / g] = (uint8_t)(int8_t)Z;
                }
                int32_t q = code_of((float)W[j], Sb, Z, qmin, qmax);
                store_code(codes, N, K, bits, n, j, q);
                double w_hat = (double)qzo_bf16_to_f32(Sb) * (double)(q - Z);
                double e = (W[j] - w_hat) / U[j * K + j];
                E[j - i] = e;
                W[j] = w_hat;
                for (int64_t k = j + 1; k < end; ++k) W[k] -= e * U[j * K + k];
            }
            /* the block is done: one update of every later column */
            for (int64_t k = end; k < K; ++k) {
                double v = 0.0;
                for (int64_t j = i; j < end; ++j) v += E[j - i] * U[j * K + k];
                W[k] -= v;
            }
        }
        if (w_out)
            for (int64_t k = 0; k < K; ++k) w_out[n * K + k] = W[k];
        free(W); free(E); free(grp);
    }
    return failed ? -1 : 0;
}

/* The whole layer: Hessian from the calibration samples, damping, factor,
 * then the column loop (see above). */
int qzo_gptq_quantize(const float *w, const uint16_t *x, int64_t N, int64_t K,
                      int64_t n_samples, double damp, int64_t block, int bits, int symmetric,
                      int64_t g, uint8_t *codes, uint16_t *scales, uint8_t *zeros)
{
    double *H = (double *)malloc((size_t)(K * K) * sizeof(double));
    double *U = (double *)calloc((size_t)(K * K), sizeof(double));
    int rc = -1;
    if (H && U && qzo_gptq_hessian_factor(x, K, n_samples, damp, H, U) == 0)
        rc = qzo_gptq_quantize_with_factor(w, U, N, K, block, bits, symmetric, g, codes,
                                           scales, zeros, NULL);
    free(H);
    free(U);
    return rc;
}

/* Thread control for the timed CPU baseline. */
void qzo_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int qzo_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
