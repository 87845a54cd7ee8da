/*
 * q4_0_oracle.c -- plain, slow, single-threaded float64 oracle for the Q4_0
 * weight-only dequantize-and-matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may build, load or call this file.  The
 * product library (bit_weight_only_matmul_b200) never links, imports or
 * falls back to it, and it shares no code, header, table or constant with the
 * CUDA sources.
 *
 * What it computes (the plain definition, no blocking or reordering):
 *
 *   Q4_0 block (GGUF convention): 32 consecutive weights of one row along K,
 *   stored as 18 bytes = an IEEE fp16 scale d (little-endian) followed by 16
 *   bytes qs; byte j of qs holds code q[j] in its low nibble and q[j+16] in
 *   its high nibble.  Blocks of a row are contiguous, rows follow each other.
 *   Each weight is w = (q - 8) * d.
 *     Sources: voxtral-mini-realtime-rs (Shannon-Prime fork) README,
 *     "RTF Benchmark Results" (the model is a Q4_0 GGUF); hakusoku.com story
 *     5135, section on linear ops and embeddings (a custom fused
 *     dequant+matmul shader runs the Q4 linears).  The byte layout and the
 *     (q - 8) * d rule are the GGUF Q4_0 convention, which the pages name but
 *     do not print: that reading is pinned by hand-built golden blocks in
 *     tests/golden/.
 *
 *   Y[m,n] = sum_k X[m,k] * w[n,k]   (X bf16 [M,K] row-major, W [N,K] in
 *   Q4_0 blocks, i.e. Y = X * dequant(W)^T), summed in float64 in increasing
 *   k, and the per-element tolerance scale B[m,n] = sum_k |X[m,k] * w[n,k]|.
 *
 * Every product (q-8)*d*x is exact in float64 (4 + 11 + 8 significant bits).
 *
 * Operations around the product (the steps next to it in a decoder, not the
 * hot path itself):
 *   swiglu   -- the activation between the fused gate/up projection and the
 *               down projection of a decoder layer's feed-forward block:
 *               out = silu(g) * u with silu(g) = g / (1 + exp(-g)), in
 *               float64 (the pages name the fused gate/up projection,
 *               voxtral-mini-realtime-rs (Shannon-Prime fork) README, TTS
 *               section, optimizations; the SwiGLU form of the Mistral-family
 *               feed-forward block is the reading taken, not printed there);
 *   residual -- Y + R, the residual connection after the O and down
 *               projections (same reading);
 *   gather   -- rows ids[t] of a Q4_0 matrix W[V, D] dequantized to float32:
 *               the Q4 embedding lookup the pages run on the CPU instead of
 *               keeping a 1.5 GiB fp32 table (hakusoku.com story 5135, linear
 *               ops and embeddings; voxtral-mini-realtime-rs README, "WASM
 *               Constraints Solved", item 3).  An id outside [0, V) gives a
 *               row of zeros (the pages do not say; reading of this library).
 *   quantize -- float32 weights to Q4_0 blocks by the GGUF Q4_0 rule, which
 *               the pages use offline (their quantize_tts_gguf.py, named in
 *               the voxtral-mini-realtime-rs README, TTS section) but do not
 *               print: per block of 32, m = the value of largest magnitude
 *               (the first one on ties), d = m / -8, id = 1/d (0 if d == 0),
 *               q = min(15, trunc(x * id + 8.5)), all in float32 with no
 *               fused multiply-add; the block stores fp16(d), rounded to
 *               nearest even.  Inputs must be finite.
 *
 * ORACLE_MUTANT: when compiled with -DORACLE_MUTANT=<n> (n >= 1) one
 * deliberate mistake is planted so that the pin tests can show they catch it.
 * The default build (no macro) is the oracle.
 */
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#include <math.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/* IEEE 754 binary16 -> double, by bit arithmetic (sign, 5-bit exponent with
 * bias 15, 10-bit fraction; exponent 0 = subnormal, 31 = inf/nan). */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
#if ORACLE_MUTANT == 5
    const int bias = 14; /* planted: wrong exponent bias */
#else
    const int bias = 15;
#endif
    if (e == 0) {
        v = ldexp((double)f, 1 - bias - 10);
    } else if (e == 31) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + f), e - bias - 10);
    }
    return sign ? -v : v;
}

/* bfloat16 -> double: bf16 is the upper half of an IEEE binary32 (sign,
 * 8-bit exponent with bias 127, 7-bit fraction). */
double oracle_bf16_to_double(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int e = (b >> 7) & 0xff;
    int f = b & 0x7f;
    double v;
    if (e == 0) {
        v = ldexp((double)f, 1 - 127 - 7);
    } else if (e == 255) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(128 + f), e - 127 - 7);
    }
    return sign ? -v : v;
}

/* Bytes of one Q4_0 row of K weights (K a multiple of 32). */
int64_t oracle_q4_0_row_bytes(int64_t K)
{
    return (K / 32) * 18;
}

/* Pack codes q[N,K] (low nibble of each byte is used) and fp16 scale bits
 * d[N,K/32] into Q4_0 blocks W (N * K/32 * 18 bytes). */
void oracle_q4_0_pack(const uint8_t *codes, const uint16_t *scales, uint8_t *W,
                      int64_t N, int64_t K)
{
    int64_t nb = K / 32;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t b = 0; b < nb; b++) {
            uint8_t *blk = W + (n * nb + b) * 18;
            const uint8_t *q = codes + n * K + b * 32;
            uint16_t d = scales[n * nb + b];
            blk[0] = (uint8_t)(d & 0xff);
            blk[1] = (uint8_t)(d >> 8);
            for (int j = 0; j < 16; j++) {
                uint8_t lo = q[j] & 0x0f;
                uint8_t hi = q[j + 16] & 0x0f;
#if ORACLE_MUTANT == 1
                blk[2 + j] = (uint8_t)(hi | (lo << 4)); /* planted: nibbles swapped */
#else
                blk[2 + j] = (uint8_t)(lo | (hi << 4));
#endif
            }
        }
    }
}

/* Inverse of pack: recover codes (0..15) and fp16 scale bits from W. */
void oracle_q4_0_unpack(const uint8_t *W, uint8_t *codes, uint16_t *scales,
                        int64_t N, int64_t K)
{
    int64_t nb = K / 32;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t b = 0; b < nb; b++) {
            const uint8_t *blk = W + (n * nb + b) * 18;
            uint8_t *q = codes + n * K + b * 32;
            scales[n * nb + b] = (uint16_t)(blk[0] | (blk[1] << 8));
            for (int j = 0; j < 16; j++) {
                q[j] = blk[2 + j] & 0x0f;
                q[j + 16] = blk[2 + j] >> 4;
            }
        }
    }
}

/* One dequantized weight w[n,k] = (q - 8) * d, read straight from W. */
static double q4_0_weight(const uint8_t *W, int64_t K, int64_t n, int64_t k)
{
    int64_t nb = K / 32;
    int64_t b = k / 32;
    int j = (int)(k % 32);
    const uint8_t *blk = W + (n * nb + b) * 18;
    double d = oracle_half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
    int q = (j < 16) ? (blk[2 + j] & 0x0f) : (blk[2 + j - 16] >> 4);
#if ORACLE_MUTANT == 2
    return (double)(q - 7) * d; /* planted: wrong zero point */
#elif ORACLE_MUTANT == 3
    return (double)(8 - q) * d; /* planted: wrong sign */
#else
    return (double)(q - 8) * d;
#endif
}

/* Dequantize W[N,K] to float64 (exact). */
void oracle_q4_0_dequant_f64(const uint8_t *W, double *out, int64_t N, int64_t K)
{
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++)
            out[n * K + k] = q4_0_weight(W, K, n, k);
}

/* Dequantize W[N,K] to float32.  (q-8)*d has at most 15 significant bits and
 * lies within the float32 range, so this is exact and well defined for a
 * bit-exact comparison. */
void oracle_q4_0_dequant_f32(const uint8_t *W, float *out, int64_t N, int64_t K)
{
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++)
            out[n * K + k] = (float)q4_0_weight(W, K, n, k);
}

/* Y[m,n] for one (m,n): sum over k in increasing order, float64, and the
 * tolerance scale B[m,n] = sum |x*w|. */
static void q4_0_dot(const uint8_t *W, const uint16_t *X, int64_t K, int64_t m,
                     int64_t n, double *y, double *bound)
{
    double s = 0.0, a = 0.0;
#if ORACLE_MUTANT == 4
    int64_t kend = K - 32; /* planted: last block of the row dropped */
#else
    int64_t kend = K;
#endif
    for (int64_t k = 0; k < kend; k++) {
        double x = oracle_bf16_to_double(X[m * K + k]);
        double w = q4_0_weight(W, K, n, k);
        s += x * w;
        a += fabs(x * w);
    }
    *y = s;
    *bound = a;
}

/* Full product: Y[M,N] (float64) and B[M,N]. */
void oracle_q4_0_gemm(const uint8_t *W, const uint16_t *X, double *Y, double *B,
                      int64_t M, int64_t N, int64_t K)
{
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
#if ORACLE_MUTANT == 6
            q4_0_dot(W, X, K, m, n, &Y[n * M + m], &B[n * M + m]); /* planted: output transposed */
#else
            q4_0_dot(W, X, K, m, n, &Y[m * N + n], &B[m * N + n]);
#endif
        }
}

/* Selected outputs only: Y[i] = Y[ms[i], ns[i]] (for full-size checks where
 * the whole product is too slow on one core). */
void oracle_q4_0_gemm_sampled(const uint8_t *W, const uint16_t *X, int64_t M,
                              int64_t N, int64_t K, const int64_t *ms,
                              const int64_t *ns, int64_t count, double *Y,
                              double *B)
{
    (void)M;
    (void)N;
    for (int64_t i = 0; i < count; i++)
        q4_0_dot(W, X, K, ms[i], ns[i], &Y[i], &B[i]);
}

/* Rows ids[0..T) of W[V, D] (Q4_0) dequantized to float32 (exact); an id
 * outside [0, V) gives a row of zeros.  Returns the number of such ids. */
int64_t oracle_q4_0_gather_f32(const uint8_t *W, const int32_t *ids, float *out,
                               int64_t T, int64_t V, int64_t D)
{
    int64_t bad = 0;
    for (int64_t t = 0; t < T; t++) {
#if ORACLE_MUTANT == 7
        int64_t v = (int64_t)ids[t] + 1; /* planted: off-by-one row */
#else
        int64_t v = (int64_t)ids[t];
#endif
        for (int64_t k = 0; k < D; k++) {
            if (v < 0 || v >= V)
                out[t * D + k] = 0.0f;
            else
                out[t * D + k] = (float)q4_0_weight(W, D, v, k);
        }
        if (v < 0 || v >= V)
            bad++;
    }
    return bad;
}

/* IEEE binary32 -> binary16 bits, rounding to nearest, ties to even, by bit
 * arithmetic: overflow gives +-inf, NaN stays NaN (quiet), values below half
 * the smallest subnormal give +-0. */
uint16_t oracle_float_to_half(float f)
{
    uint32_t x;
    memcpy(&x, &f, 4);
    uint32_t sign = (x >> 16) & 0x8000u;
    int32_t exp = (int32_t)((x >> 23) & 0xffu);
    uint32_t man = x & 0x7fffffu;
    if (exp == 0xff)
        return (uint16_t)(sign | 0x7c00u | (man ? 0x200u : 0u));
    int32_t e = exp - 127 + 15;              /* biased binary16 exponent */
    if (e >= 31)
        return (uint16_t)(sign | 0x7c00u);
    if (e <= 0) {                            /* binary16 subnormal or zero */
        if (e < -10)
            return (uint16_t)sign;
        uint32_t full = man | 0x800000u;     /* 24-bit significand */
        int shift = 14 - e;                  /* 14 .. 24 */
        uint32_t hm = full >> shift;
        uint32_t rem = full & ((1u << shift) - 1u);
        uint32_t half = 1u << (shift - 1);
        if (rem > half || (rem == half && (hm & 1u)))
            hm++;                            /* may carry into the smallest normal */
        return (uint16_t)(sign | hm);
    }
    uint32_t h = sign | ((uint32_t)e << 10) | (man >> 13);
    uint32_t rem = man & 0x1fffu;
    if (rem > 0x1000u || (rem == 0x1000u && (h & 1u)))
        h++;                                 /* a carry moves into the exponent, up to inf */
    return (uint16_t)h;
}

/* X[N, K] float32 -> W (Q4_0), K a multiple of 32, by the rule in the header. */
void oracle_q4_0_quantize(const float *X, uint8_t *W, int64_t N, int64_t K)
{
    int64_t nb = K / 32;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t b = 0; b < nb; b++) {
            const float *x = X + n * K + b * 32;
            float amax = 0.0f, m = 0.0f;
            for (int j = 0; j < 32; j++) {
                float a = fabsf(x[j]);
#if ORACLE_MUTANT == 9
                if (amax <= a) { /* planted: the last of equal magnitudes wins */
#else
                if (amax < a) {
#endif
                    amax = a;
                    m = x[j];
                }
            }
#if ORACLE_MUTANT == 8
            float d = m / 8.0f; /* planted: scale sign flipped */
#else
            float d = m / -8.0f;
#endif
            float id = (d != 0.0f) ? 1.0f / d : 0.0f;
            uint8_t q[32];
            for (int j = 0; j < 32; j++) {
                volatile float p = x[j] * id;   /* separate rounding of the product */
#if ORACLE_MUTANT == 10
                float v = p + 8.0f;             /* planted: truncation, not rounding */
#else
                float v = p + 8.5f;
#endif
                int c = (int)v;                 /* v >= 0 for finite inputs: truncation */
                q[j] = (uint8_t)(c > 15 ? 15 : c);
            }
            uint16_t dh = oracle_float_to_half(d);
            uint8_t *blk = W + (n * nb + b) * 18;
            blk[0] = (uint8_t)(dh & 0xff);
            blk[1] = (uint8_t)(dh >> 8);
            for (int j = 0; j < 16; j++)
                blk[2 + j] = (uint8_t)((q[j] & 0x0f) | ((q[j + 16] & 0x0f) << 4));
        }
    }
}

/* out[i] = silu(g[i]) * u[i], silu(g) = g / (1 + exp(-g)), float64. */
void oracle_swiglu(const double *g, const double *u, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; i++) {
#if ORACLE_MUTANT == 11
        double s = g[i] / (1.0 + exp(g[i])); /* planted: wrong sign in the exponent */
#else
        double s = g[i] / (1.0 + exp(-g[i]));
#endif
        out[i] = s * u[i];
    }
}
