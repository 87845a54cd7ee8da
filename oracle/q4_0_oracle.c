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
 * ORACLE_MUTANT: when compiled with -DORACLE_MUTANT=<n> (n >= 1) one
 * deliberate mistake is planted so that the pin tests can show they catch it.
 * The default build (no macro) is the oracle.
 */
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#include <math.h>

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
