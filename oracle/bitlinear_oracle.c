/*
 * bitlinear_oracle.c -- plain, slow CPU oracle for the BitLinear W1.58A8 forward.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this file's library.  The CUDA
 * library shares no code, header, table or constant with it.
 *
 * Built with gcc -O2 -fno-fast-math -ffp-contract=off (SSE arithmetic on
 * x86-64, so every float operation below is one IEEE binary32 operation with
 * round-to-nearest-even, and nothing is fused into an FMA).  A second build of
 * the same source with -fopenmp (liboracle_omp.so) only shares the integer
 * contraction's (m, n) pairs among threads; it exists for the benchmark's
 * all-core CPU baseline.
 *
 * Sources (web pages on ternary-weight linear layers):
 *   [MMF]  DataCamp blog "MatMul-free language models" (Dutch), section
 *          "MatMul vervangen door ternaire bewerkingen": absmean scales the
 *          weight matrix by its mean absolute value and rounds every element
 *          to the nearest of -1, 0, +1; a multiply by -1/0/+1 becomes a
 *          negate / zero / pass-through.
 *   [BNC]  unite.ai "Microsofts Inference Framework bringt 1-Bit grosse
 *          Sprachmodelle auf lokale Geraete" (German), section "Mathematische
 *          Grundlagen": eq. 2 "Aktivierungsquantisierung" (absmax quantiser
 *          with Q_b and gamma = ||x||_inf) and eq. 3 "BitLinear-Betrieb"
 *          (y = W_f x_hat (beta gamma / Q_b)); the 1-bit variant of the
 *          weights is item 1 "Gewichtsbinarisierung", eq. 1
 *          (W_f = Sign(W - alpha), alpha = mean(W)).
 *
 * Readings taken where the pages are silent (each one is listed with its
 * reason in the design notes of the repository):
 *   - beta is one scale per matrix, the exact mean of |W| rounded once to
 *     binary64 and then once to binary32; eps = 1e-5 is added only in the
 *     divisor of the ternariser.
 *   - "round" is round-half-to-even; ternary codes are clip(rint(q), -1, 1).
 *   - Q_b = 127 with a symmetric clamp to [-127, 127]; gamma is per token,
 *     floored at 1e-5; the scale s = 127 / gamma is formed first, x * s after.
 *   - the output is y = (float)acc * ((beta * gamma) / 127) in binary32.
 *   - binary variant: alpha is the exact mean of W rounded like beta;
 *     Sign(0) = -1 as the page's definition of Sign states; beta of a
 *     binarised matrix is the same absmean scale (the page names beta a
 *     scaling factor without a formula).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Exact sum of |w| over n binary32 values, correctly rounded to binary64.   */
/*                                                                           */
/* Every finite binary32 magnitude is an integer multiple of 2^-149: its     */
/* 24-bit significand m times 2^(e-150) for biased exponent e >= 1, or the   */
/* 23-bit fraction times 2^-149 when e == 0.  The sum is therefore an        */
/* integer in units of 2^-149, kept here in 32-bit digits (one per uint64    */
/* limb, so carries can wait until the end).  Nothing is rounded until the   */
/* final conversion.                                                         */
/* ------------------------------------------------------------------------ */
#define ORC_LIMBS 12  /* 12 * 32 = 384 bits >= 278 value bits + 64 carry bits */

/* Add the magnitude of the binary32 pattern u (sign ignored) to acc. */
static void limbs_add(uint64_t acc[ORC_LIMBS], uint32_t u)
{
    u &= 0x7FFFFFFFu;
    if (u == 0) return;
    uint32_t e = u >> 23;
    uint64_t m = u & 0x7FFFFFu;
    uint32_t pos;                               /* bit position of m's bit 0 */
    if (e == 0) { pos = 0; }
    else { m |= 0x800000u; pos = e - 1; }
    uint64_t shifted = m << (pos % 32);         /* < 2^55 */
    uint32_t d = pos / 32;
    acc[d] += shifted & 0xFFFFFFFFu;
    acc[d + 1] += shifted >> 32;
}

/* carry-normalise to 32-bit digits */
static void limbs_normalise(uint64_t acc[ORC_LIMBS])
{
    for (int d = 0; d + 1 < ORC_LIMBS; ++d) {
        acc[d + 1] += acc[d] >> 32;
        acc[d] &= 0xFFFFFFFFu;
    }
}

/* The normalised integer acc (units of 2^-149), rounded once to binary64. */
static double limbs_to_double(const uint64_t acc[ORC_LIMBS])
{
    int top = -1;
    for (int d = ORC_LIMBS - 1; d >= 0; --d)
        if (acc[d]) { top = d; break; }
    if (top < 0) return 0.0;
    /* highest set bit of the whole integer */
    int hb = 31;
    while (!((acc[top] >> hb) & 1u)) --hb;
    int msb = top * 32 + hb;
    /* take bits [msb-63, msb] into t, OR every lower bit into t's bit 0 */
    uint64_t t = 0;
    int lo = msb - 63;
    for (int b = 63; b >= 0; --b) {
        int p = lo + b;
        uint64_t bit = (p >= 0) ? ((acc[p / 32] >> (p % 32)) & 1u) : 0u;
        t |= bit << b;
    }
    int sticky = 0;
    for (int p = 0; p < lo; ++p)
        if ((acc[p / 32] >> (p % 32)) & 1u) { sticky = 1; break; }
    if (sticky) t |= 1u;
    /* (double)t rounds to nearest even; bit 0 of t carries the sticky bit,
       which sits 11 places below t's rounding position. */
    double d = (double)t;
    return ldexp(d, lo - 149);
}

double orc_exact_abs_sum(const float* w, int64_t n)
{
    uint64_t acc[ORC_LIMBS];
    memset(acc, 0, sizeof acc);
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u;
        memcpy(&u, &w[i], 4);
        limbs_add(acc, u);
    }
    limbs_normalise(acc);
    return limbs_to_double(acc);
}

/* Exact signed sum of n binary32 values, correctly rounded to binary64: the
 * positive and the negative elements are added exactly into two integers, the
 * smaller magnitude is subtracted from the larger, and the difference is
 * rounded once. */
double orc_exact_sum(const float* w, int64_t n)
{
    uint64_t pos[ORC_LIMBS], neg[ORC_LIMBS];
    memset(pos, 0, sizeof pos);
    memset(neg, 0, sizeof neg);
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u;
        memcpy(&u, &w[i], 4);
        limbs_add((u >> 31) ? neg : pos, u);
    }
    limbs_normalise(pos);
    limbs_normalise(neg);
    int cmp = 0;
    for (int d = ORC_LIMBS - 1; d >= 0 && cmp == 0; --d)
        cmp = pos[d] > neg[d] ? 1 : pos[d] < neg[d] ? -1 : 0;
    if (cmp == 0) return 0.0;
    const uint64_t* big = cmp > 0 ? pos : neg;
    const uint64_t* small = cmp > 0 ? neg : pos;
    uint64_t diff[ORC_LIMBS];
    uint64_t borrow = 0;
    for (int d = 0; d < ORC_LIMBS; ++d) {
        uint64_t sub = small[d] + borrow;           /* digits < 2^32: no wrap */
        borrow = big[d] < sub ? 1u : 0u;
        diff[d] = (big[d] + (borrow << 32)) - sub;
    }
    double r = limbs_to_double(diff);
    return cmp > 0 ? r : -r;
}

/* [MMF] absmean: beta = mean |W| over the whole matrix (one scale per matrix). */
float orc_absmean_beta(const float* W, int64_t N, int64_t K)
{
    int64_t n = N * K;
    if (n <= 0) return 0.0f;
    double s = orc_exact_abs_sum(W, n);
    return (float)(s / (double)n);
}

/* [MMF] absmean ternarisation: W_t = clip(round(W / (beta + eps)), -1, 1). */
void orc_ternarize(const float* W, int64_t N, int64_t K, float beta, float eps, int8_t* W_t)
{
    float den = beta + eps;
    for (int64_t i = 0; i < N * K; ++i) {
        float q = W[i] / den;
        float r = rintf(q);               /* nearest, ties to even */
        if (r > 1.0f) r = 1.0f;
        if (r < -1.0f) r = -1.0f;
        W_t[i] = (int8_t)r;
    }
}

/* [BNC] "Mathematische Grundlagen", item 1 "Gewichtsbinarisierung", eq. 1:
 * alpha = mean(W) over the whole matrix -- the exact sum rounded once to
 * binary64, divided by N*K in binary64, rounded to binary32 (as beta). */
float orc_mean_alpha(const float* W, int64_t N, int64_t K)
{
    int64_t n = N * K;
    if (n <= 0) return 0.0f;
    double s = orc_exact_sum(W, n);
    return (float)(s / (double)n);
}

/* [BNC] eq. 1: W_b = Sign(W - alpha), with Sign(d) = +1 for d > 0 and -1
 * otherwise (zero included); d = W - alpha is one binary32 subtraction. */
void orc_binarize(const float* W, int64_t N, int64_t K, float alpha, int8_t* W_b)
{
    for (int64_t i = 0; i < N * K; ++i) {
        float d = W[i] - alpha;
        W_b[i] = d > 0.0f ? (int8_t)1 : (int8_t)-1;
    }
}

/* 1-bit storage of binary weights, 32 per uint32: for row n and word j, the
 * weight at k = 32j + 4s + b (s in 0..7, b in 0..3) is bit 8b + s of
 * W_p[n, j], set for +1 and clear for -1 (any w <= 0 is stored as -1). */
void orc_pack_bits(const int8_t* W_b, int64_t N, int64_t K, uint32_t* W_p)
{
    int64_t KW = K / 32;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < KW; ++j) {
            uint32_t word = 0;
            for (int t = 0; t < 32; ++t) {
                int s = t / 4, b = t % 4;
                if (W_b[n * K + 32 * j + t] > 0) word |= 1u << (8 * b + s);
            }
            W_p[n * KW + j] = word;
        }
}

/* Inverse of orc_pack_bits: set bits give +1, clear bits -1. */
void orc_unpack_bits(const uint32_t* W_p, int64_t N, int64_t K, int8_t* W_b)
{
    int64_t KW = K / 32;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < KW; ++j) {
            uint32_t word = W_p[n * KW + j];
            for (int t = 0; t < 32; ++t) {
                int s = t / 4, b = t % 4;
                W_b[n * K + 32 * j + t] = ((word >> (8 * b + s)) & 1u) ? (int8_t)1 : (int8_t)-1;
            }
        }
}

/* 2-bit storage of the trits (the "1.58 bit" weights of [BNC] "Ternaeres
 * Gewichtssystem", stored in 2 bits): code c = w + 1 in {0, 1, 2}; for row n
 * and word j, the trit at k = 16j + 4s + b occupies bits [8b + 2s, 8b + 2s + 1]. */
void orc_pack(const int8_t* W_t, int64_t N, int64_t K, uint32_t* W_p)
{
    int64_t KW = K / 16;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < KW; ++j) {
            uint32_t word = 0;
            for (int t = 0; t < 16; ++t) {
                int s = t / 4, b = t % 4;
                uint32_t c = (uint32_t)(W_t[n * K + 16 * j + t] + 1);
                word |= c << (8 * b + 2 * s);
            }
            W_p[n * KW + j] = word;
        }
}

/* Inverse of orc_pack.  Returns the number of code-3 fields met (invalid). */
int64_t orc_unpack(const uint32_t* W_p, int64_t N, int64_t K, int8_t* W_t)
{
    int64_t KW = K / 16, bad = 0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < KW; ++j) {
            uint32_t word = W_p[n * KW + j];
            for (int t = 0; t < 16; ++t) {
                int s = t / 4, b = t % 4;
                uint32_t c = (word >> (8 * b + 2 * s)) & 3u;
                if (c == 3u) ++bad;
                W_t[n * K + 16 * j + t] = (int8_t)((int)c - 1);
            }
        }
    return bad;
}

/* [BNC] eq. 2, per token: gamma = max(||x_m||_inf, 1e-5); s = 127 / gamma;
 * x_hat = clip(rint(x * s), -127, 127). */
void orc_quant_act(const float* x, int64_t M, int64_t K, int8_t* x_q, float* gamma)
{
    for (int64_t m = 0; m < M; ++m) {
        const float* row = x + m * K;
        float g = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(row[k]);
            if (a > g) g = a;
        }
        if (g < 1e-5f) g = 1e-5f;
        float s = 127.0f / g;
        for (int64_t k = 0; k < K; ++k) {
            float r = rintf(row[k] * s);
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            x_q[m * K + k] = (int8_t)r;
        }
        gamma[m] = g;
    }
}

/* [MMF] multiply by -1 / 0 / +1 becomes subtract / skip / add: the ternary
 * contraction acc[m, n] = sum_k W_t[n, k] * x_hat[m, k], written literally. */
void orc_ternary_acc(const int8_t* x_q, int64_t M, int64_t K, const int8_t* W_t, int64_t N, int32_t* acc)
{
    /* Every (m, n) is independent; an OpenMP build (the benchmark's all-core
     * CPU baseline) shares them out, a plain build ignores the pragma. */
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            const int8_t* xr = x_q + m * K;
            const int8_t* wr = W_t + n * K;
            int32_t a = 0;
            for (int64_t k = 0; k < K; ++k) {
                if (wr[k] == 1) a += xr[k];
                else if (wr[k] == -1) a -= xr[k];
                /* wr[k] == 0: skip */
            }
            acc[m * N + n] = a;
        }
}

/* [BNC] eq. 3 rescale in binary32, fixed operation order:
 * f_m = (beta * gamma_m) / 127, then y = (float)acc * f_m. */
void orc_rescale_f32(const int32_t* acc, int64_t M, int64_t N, float beta, const float* gamma, float* y)
{
    for (int64_t m = 0; m < M; ++m) {
        float f = (beta * gamma[m]) / 127.0f;
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = (float)acc[m * N + n] * f;
    }
}

/* [BNC] eq. 3 rescale carried out in binary64 (the tolerance reference). */
void orc_rescale_f64(const int32_t* acc, int64_t M, int64_t N, float beta, const float* gamma, double* y)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = (double)acc[m * N + n] * (double)beta * (double)gamma[m] / 127.0;
}

/* binary32 -> bfloat16, round to nearest, ties to even (finite inputs). */
void orc_f32_to_bf16(const float* y, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u;
        memcpy(&u, &y[i], 4);
        uint32_t lsb = (u >> 16) & 1u;
        out[i] = (uint16_t)((u + 0x7FFFu + lsb) >> 16);
    }
}

/* RMSNorm scalar (gain 1) of a token, [MMF] figure item "RMS norm": the
 * activations are normalised before quantisation.  rho = 1 / sqrt(mean(x^2) + eps),
 * evaluated in binary64 and rounded once to binary32. */
float orc_rms_rho(const float* x, int64_t K, double eps)
{
    double s = 0.0;
    for (int64_t k = 0; k < K; ++k) s += (double)x[k] * (double)x[k];
    return (float)(1.0 / sqrt(s / (double)K + eps));
}

/* SiLU(gate) * up in binary64, rounded once to binary32. */
void orc_silu_mul(const float* gate, const float* up, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; ++i) {
        double g = (double)gate[i];
        double s = g / (1.0 + exp(-g));
        out[i] = (float)(s * (double)up[i]);
    }
}
