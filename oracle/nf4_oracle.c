/*
 * nf4_oracle.c -- plain, slow CPU oracle for blockwise NF4 + double quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header, table or constant generator with
 * the CUDA library; the two meet only on the byte format they both write.
 *
 * Sources (QLoRA, Dettmers et al., arXiv:2305.14314, as summarised on the
 * pages gathered for this method):
 *   - automatone "QLoRA paper explained", section "How it works", paragraph
 *     "4-bit NormalFloat (NF4)": the 16 levels sit at quantiles of a standard
 *     normal distribution.
 *   - creativeworksofknowledge "QLoRA: Fine-Tune 70B on One GPU", section
 *     "1. NF4 (NormalFloat4) quantization": levels allocated in proportion to
 *     the Gaussian, denser near zero.
 *   - HackerPapers snippet (TorchLean thread): NF4 builds on quantile
 *     quantization.
 *   - automatone, paragraph "Double Quantization (DQ)": block-wise
 *     quantization gives one scaling constant per block; DQ quantizes those
 *     constants again.
 *   - creativeworksofknowledge, section "2. Double quantization": the
 *     constants go FP32 -> FP8.
 *   - automatone, section "How it works", first paragraph: weights are
 *     dequantized to the BFloat16 compute type on the fly.
 * Block size 64 for the weights and 256 for the constants, mean subtraction
 * before the second quantization, a codebook with an exact zero: these come
 * from the benchmark spec of this hot path, not from the pages.
 *
 * Readings where the pages are silent:
 *   R1  codebook: 8 positive quantiles Phi^-1(1/2 + (delta-1/2) j/8), j=1..8,
 *       7 negative ones -Phi^-1(1/2 + (delta-1/2) j/7), j=1..7, plus 0, each
 *       side divided by Phi^-1(delta); delta = 1 - (1/30 + 1/32)/2.
 *       Computed in double, rounded once to float.
 *   R2  nearest level in exact arithmetic; a tie goes to the lower index.
 *   R3  codes are chosen against the exact block absmax c1 (float division
 *       x / c1), not against the double-quantized constant.
 *   R4  packing: byte j holds element 2j in its high nibble and element 2j+1
 *       in its low nibble; a ragged tail is padded with the zero code.
 *   R5  mean mu = float(double-sum(c1) / count) over the whole tensor;
 *       c2 = max |c1 - mu| per group of 256 constants (float subtraction);
 *       q = E4M3(RNE(float(float((c1 - mu) / c2) * 448))); q = 0 if c2 == 0.
 *       FP8 is OCP E4M3 "fn" (max 448, no infinities).
 *   R6  dequant: c1' = fmaf(e4m3(q), c2 / 448, mu); w' = bf16_RNE(L[code]*c1').
 *       Without double quantization the constant is c1 itself (fp32).
 *   R7  the comparison types INT4 and FP4 (see nf4o_levels); the encode,
 *       packing and constants are the same for every type.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -fPIC
 * -shared.  FP contraction is off so every float operation rounds once, as
 * written.  OpenMP only splits independent blocks; it never reorders a sum.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define NF4O_EXPORT __attribute__((visibility("default")))

/* ---------------------------------------------------------------------- */
/* Scalar formats.                                                        */
/* ---------------------------------------------------------------------- */

/* bf16 bit pattern -> float (exact: bf16 is the top half of a float). */
NF4O_EXPORT float nf4o_bf16_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* float -> bf16, round to nearest, ties to even, from the definition:
 * pick the exponent of |x|, divide by that binade's bf16 quantum (a power of
 * two, so exact in double), round the quotient to an integer with rint()
 * (default mode: nearest-even), rebuild.  bf16 keeps 7 fraction bits and the
 * float exponent range; subnormals have quantum 2^-133. */
NF4O_EXPORT uint16_t nf4o_bf16_rne(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    if (isnan(x)) return (uint16_t)(sign | 0x7FC0u);
    double a = fabs((double)x);
    if (isinf(x)) return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0) return sign;
    int e2;
    (void)frexp(a, &e2);            /* a = m * 2^e2, m in [0.5, 1) */
    int e = e2 - 1;                 /* a in [2^e, 2^(e+1)) */
    if (e < -126) e = -126;         /* subnormal binade shares min-normal quantum */
    double quantum = ldexp(1.0, e - 7);
    double q = rint(a / quantum);   /* integer significand, 0..256 */
    double r = q * quantum;         /* rounded magnitude, exact */
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);   /* overflow -> inf */
    float rf = (float)r;            /* exact: r is a bf16 value */
    uint32_t ru;
    memcpy(&ru, &rf, 4);
    return (uint16_t)(sign | (ru >> 16));
}

/* OCP E4M3 ("fn") byte -> float.  Bias 7; exponent field 0 is subnormal with
 * quantum 2^-9; S.1111.111 is NaN; there is no infinity. */
NF4O_EXPORT float nf4o_e4m3_to_float(uint8_t b)
{
    int s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

/* float -> E4M3, round to nearest, ties to even, from the definition.
 * Magnitudes that round above 448 saturate to 448 (the double-quant path
 * never produces them: |t * 448| <= 448). */
NF4O_EXPORT uint8_t nf4o_e4m3_rne(float x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    if (isnan(x)) return (uint8_t)(sign | 0x7F);
    double a = fabs((double)x);
    if (a == 0.0) return sign;
    int e2;
    (void)frexp(a, &e2);
    int e = e2 - 1;                 /* a in [2^e, 2^(e+1)) */
    if (e < -6) e = -6;             /* subnormals: quantum 2^-9 */
    double quantum = ldexp(1.0, e - 3);
    double q = rint(a / quantum);
    double r = q * quantum;
    if (r > 448.0) r = 448.0;
    /* re-encode r (an exact E4M3 magnitude) */
    if (r < ldexp(1.0, -6)) {
        int m = (int)(r / ldexp(1.0, -9));
        return (uint8_t)(sign | m);
    }
    (void)frexp(r, &e2);
    e = e2 - 1;
    int m = (int)(r / ldexp(1.0, e - 3)) - 8;
    return (uint8_t)(sign | ((e + 7) << 3) | m);
}

/* ---------------------------------------------------------------------- */
/* R1: the NF4 codebook.                                                  */
/* ---------------------------------------------------------------------- */

static double std_normal_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* Phi^-1(p) for p in (0, 1) by plain bisection on the CDF.  Slow and exact
 * to the last bit the CDF can resolve. */
NF4O_EXPORT double nf4o_normal_quantile(double p)
{
    double lo = -40.0, hi = 40.0;
    for (int it = 0; it < 400; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid == lo || mid == hi) break;
        if (std_normal_cdf(mid) < p) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

NF4O_EXPORT double nf4o_default_delta(void) { return 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0); }

/* L[0..15] ascending: L[0] = -1, L[7] = 0, L[15] = +1. */
NF4O_EXPORT void nf4o_codebook(double delta, float L[16])
{
    double top = nf4o_normal_quantile(delta);
    for (int j = 1; j <= 7; ++j)            /* negative side: 7 levels */
        L[7 - j] = (float)(-nf4o_normal_quantile(0.5 + (delta - 0.5) * j / 7.0) / top);
    L[7] = 0.0f;
    for (int j = 1; j <= 8; ++j)            /* positive side: 8 levels */
        L[7 + j] = (float)(nf4o_normal_quantile(0.5 + (delta - 0.5) * j / 8.0) / top);
}

/* R2: index of the level nearest to n; ties go to the lower index.  The
 * differences are taken in double, where n - L[i] is exact for every n the
 * decision can depend on (|n| and |L[i]| within a few binades of each other). */
NF4O_EXPORT int nf4o_nearest(float n, const float L[16])
{
    int best = 0;
    double bd = fabs((double)n - (double)L[0]);
    for (int i = 1; i < 16; ++i) {
        double d = fabs((double)n - (double)L[i]);
        if (d < bd) { bd = d; best = i; }
    }
    return best;
}

/* ---------------------------------------------------------------------- */
/* R7: the other 4-bit data types the pages compare NF4 with.             */
/* ---------------------------------------------------------------------- */

/* automatone, "4-bit NormalFloat (NF4)": standard 4-bit integers space their
 * 16 levels evenly, 4-bit floats space theirs by exponent, and NF4 beats both
 * (also "Results": FP4 trails NF4).  Both tables are normalized to [-1, 1],
 * the range blockwise absmax scaling maps a block into.
 *
 * INT4: 16 evenly spaced levels from -1 to +1, L[i] = (2i - 15) / 15 (no
 *   exact zero: 16 even steps over a symmetric range cannot have one).
 * FP4:  the values of the 4-bit float E2M1 (1 sign bit, 2 exponent bits with
 *   bias 1, 1 mantissa bit; exponent field 0 is subnormal), decoded from each
 *   of the 16 bit patterns and divided by the largest magnitude, 6.  +0 and -0
 *   are one value, so there are 15 distinct levels: they fill L[0..14] in
 *   ascending order and L[15] repeats +1.  Code 15 is never chosen: the
 *   nearest-level rule sends a tie to the lower index. */
#define NF4O_TYPE_NF4 0
#define NF4O_TYPE_FP4 1
#define NF4O_TYPE_INT4 2

static double e2m1_decode(int bits)
{
    int s = (bits >> 3) & 1, e = (bits >> 1) & 3, m = bits & 1;
    double mag = (e == 0) ? ldexp((double)m, -1)          /* 0.m x 2^(1 - bias) */
                          : ldexp(1.0 + 0.5 * m, e - 1);  /* 1.m x 2^(e - bias) */
    return s ? -mag : mag;
}

static int cmp_double(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x > y) - (x < y);
}

NF4O_EXPORT int nf4o_levels(int type, float L[16])
{
    if (type == NF4O_TYPE_NF4) {
        nf4o_codebook(nf4o_default_delta(), L);
        return 0;
    }
    if (type == NF4O_TYPE_INT4) {
        for (int i = 0; i < 16; ++i) L[i] = (float)((2.0 * i - 15.0) / 15.0);
        return 0;
    }
    if (type == NF4O_TYPE_FP4) {
        double v[16];
        for (int b = 0; b < 16; ++b) v[b] = e2m1_decode(b);
        qsort(v, 16, sizeof(double), cmp_double);
        double top = v[15];
        int n = 0;
        for (int b = 0; b < 16; ++b)
            if (n == 0 || v[b] != v[n - 1]) v[n++] = v[b];   /* -0 == +0: one level */
        for (int i = 0; i < n; ++i)
            if (v[i] == 0.0) v[i] = 0.0;                      /* the zero level is +0 */
        for (int i = 0; i < 16; ++i) L[i] = (float)(v[i < n ? i : n - 1] / top);
        return 0;
    }
    return -1;
}

/* ---------------------------------------------------------------------- */
/* Storage sizes.                                                         */
/* ---------------------------------------------------------------------- */

/* With double quantization (bs2 > 0): one E4M3 byte per block, one float c2
 * per group of bs2 blocks and one float mean.  Without it (bs2 == 0): the
 * block absmax stored as one fp32 per block (reported in *absmax_q), no c2,
 * no mean (creativeworksofknowledge, "2. Double quantization": the constants
 * go FP32 -> FP8). */
NF4O_EXPORT void nf4o_storage_bytes(int64_t numel, int bs, int bs2,
                                    int64_t *codes, int64_t *absmax_q,
                                    int64_t *absmax_c2, int64_t *mean)
{
    int64_t nblocks = (numel + bs - 1) / bs;
    *codes = (numel + 1) / 2;
    if (bs2 == 0) {
        *absmax_q = 4 * nblocks;                /* one float per block */
        *absmax_c2 = 0;
        *mean = 0;
        return;
    }
    *absmax_q = nblocks;                       /* one FP8 byte per block */
    *absmax_c2 = 4 * ((nblocks + bs2 - 1) / bs2);   /* one float per group */
    *mean = 4;                                  /* one float per tensor */
}

/* ---------------------------------------------------------------------- */
/* Blockwise absmax NF4 encode (R2, R3, R4).                              */
/* ---------------------------------------------------------------------- */

/* w: numel bf16 patterns, flattened row-major.  packed: (numel+1)/2 bytes.
 * c1: one float per block of bs. */
NF4O_EXPORT void nf4o_encode(const uint16_t *w, int64_t numel, int bs,
                             const float L[16], uint8_t *packed, float *c1)
{
    int64_t nblocks = (numel + bs - 1) / bs;
    int64_t nbytes = (numel + 1) / 2;
    uint8_t *codes = (uint8_t *)malloc((size_t)(nblocks * bs));
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nblocks; ++b) {
        int64_t lo = b * bs, hi = lo + bs < numel ? lo + bs : numel;
        float amax = 0.0f;
        for (int64_t i = lo; i < hi; ++i) {
            float a = fabsf(nf4o_bf16_to_float(w[i]));
            if (a > amax) amax = a;
        }
        c1[b] = amax;
        for (int64_t i = lo; i < lo + bs; ++i) {
            int code = 7;                       /* the zero level */
            if (i < hi && amax > 0.0f) {
                float n = nf4o_bf16_to_float(w[i]) / amax;   /* one IEEE float division */
                code = nf4o_nearest(n, L);
            }
            codes[i] = (uint8_t)code;
        }
    }
    for (int64_t j = 0; j < nbytes; ++j) {
        uint8_t hiN = codes[2 * j];
        uint8_t loN = (2 * j + 1 < numel) ? codes[2 * j + 1] : 7;
        packed[j] = (uint8_t)((hiN << 4) | loN);
    }
    free(codes);
}

/* ---------------------------------------------------------------------- */
/* Double quantization of the block constants (R5).                       */
/* ---------------------------------------------------------------------- */

NF4O_EXPORT float nf4o_mean(const float *c1, int64_t nblocks)
{
    double s = 0.0;
    for (int64_t b = 0; b < nblocks; ++b) s += (double)c1[b];
    return (float)(s / (double)nblocks);
}

NF4O_EXPORT void nf4o_double_quant(const float *c1, int64_t nblocks, int bs2,
                                   uint8_t *q, float *c2, float *mean)
{
    float mu = nf4o_mean(c1, nblocks);
    *mean = mu;
    int64_t ngroups = (nblocks + bs2 - 1) / bs2;
    for (int64_t g = 0; g < ngroups; ++g) {
        int64_t lo = g * bs2, hi = lo + bs2 < nblocks ? lo + bs2 : nblocks;
        float m = 0.0f;
        for (int64_t b = lo; b < hi; ++b) {
            float d = fabsf(c1[b] - mu);
            if (d > m) m = d;
        }
        c2[g] = m;
        for (int64_t b = lo; b < hi; ++b) {
            if (m == 0.0f) { q[b] = 0; continue; }
            float t = (c1[b] - mu) / m;
            float scaled = t * 448.0f;
            q[b] = nf4o_e4m3_rne(scaled);
        }
    }
}

/* ---------------------------------------------------------------------- */
/* Two-level dequantization (R6).                                         */
/* ---------------------------------------------------------------------- */

NF4O_EXPORT float nf4o_block_constant(uint8_t q, float c2, float mu)
{
    return fmaf(nf4o_e4m3_to_float(q), c2 / 448.0f, mu);
}

NF4O_EXPORT void nf4o_dequant(const uint8_t *packed, const uint8_t *q,
                              const float *c2, float mu, int64_t numel,
                              int bs, int bs2, const float L[16], uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < numel; ++i) {
        int64_t b = i / bs;
        float c1p = nf4o_block_constant(q[b], c2[b / bs2], mu);
        uint8_t byte = packed[i / 2];
        int code = (i % 2 == 0) ? (byte >> 4) : (byte & 15);
        float v = L[code] * c1p;
        out[i] = nf4o_bf16_rne(v);
    }
}

/* Dequantization without double quantization: the block's fp32 absmax is
 * the constant, w' = bf16_RNE(L[code] * c1). */
NF4O_EXPORT void nf4o_dequant_f32(const uint8_t *packed, const float *c1,
                                  int64_t numel, int bs, const float L[16],
                                  uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < numel; ++i) {
        uint8_t byte = packed[i / 2];
        int code = (i % 2 == 0) ? (byte >> 4) : (byte & 15);
        float v = L[code] * c1[i / bs];
        out[i] = nf4o_bf16_rne(v);
    }
}

/* ---------------------------------------------------------------------- */
/* Array forms of the scalar roundings (used by the tests to sweep many   */
/* values without one foreign call per value).                            */
/* ---------------------------------------------------------------------- */

NF4O_EXPORT void nf4o_bf16_rne_n(const float *x, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = nf4o_bf16_rne(x[i]);
}

NF4O_EXPORT void nf4o_e4m3_rne_n(const float *x, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = nf4o_e4m3_rne(x[i]);
}
