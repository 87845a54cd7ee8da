// q4_0_convert.cuh -- register-level conversions shared by the fast kernels:
// Q4_0 codes and scale -> fp16 weights, bf16 activations -> fp16.
//
// Both use one k order inside every 32-weight block: positions 1 and 2 of
// each group of 4 swapped ((0,2), (1,3) pairs), which is the order in which a
// mask over a 32-bit word of packed codes yields nibble pairs.  Applying the
// same permutation to both operands of a dot product leaves it unchanged.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "q4_0_internal.cuh"

namespace q4dev {

// fp16 pairs of w = (q - 8) * d for one qs word v (bytes 4w .. 4w+3 of a
// block), d2 = (d, d):
//   c[0] = elements (4w, 4w+2), c[1] = (4w+1, 4w+3)        (low nibbles)
//   c[2] = elements (4w+16, 4w+18), c[3] = (4w+17, 4w+19)  (high nibbles)
// 0x6400 is fp16 1024 (10 fraction bits): 1024 + q and 1024 + 16q are exact,
// and so are (1024 + q) - 1032 and (1024 + 16q) / 16 - 72 = q - 8; the only
// rounding is the product with d (relative error <= 2^-11).
__device__ __forceinline__ void q4_word_to_fp16(uint32_t v, uint32_t d2, uint32_t (&c)[4]) {
    const uint32_t v8 = v >> 8;
    const __half2 k1032 = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
    const __half2 k16th = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
    const __half2 km72 = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));
    const __half2 d = *reinterpret_cast<const __half2 *>(&d2);
    uint32_t t[4] = {and_or(v, 0x000F000Fu, 0x64006400u), and_or(v8, 0x000F000Fu, 0x64006400u),
                     and_or(v, 0x00F000F0u, 0x64006400u), and_or(v8, 0x00F000F0u, 0x64006400u)};
    __half2 r0 = __hmul2(__hsub2(*reinterpret_cast<__half2 *>(&t[0]), k1032), d);
    __half2 r1 = __hmul2(__hsub2(*reinterpret_cast<__half2 *>(&t[1]), k1032), d);
    __half2 r2 = __hmul2(__hfma2(*reinterpret_cast<__half2 *>(&t[2]), k16th, km72), d);
    __half2 r3 = __hmul2(__hfma2(*reinterpret_cast<__half2 *>(&t[3]), k16th, km72), d);
    c[0] = *reinterpret_cast<uint32_t *>(&r0);
    c[1] = *reinterpret_cast<uint32_t *>(&r1);
    c[2] = *reinterpret_cast<uint32_t *>(&r2);
    c[3] = *reinterpret_cast<uint32_t *>(&r3);
}

// bf16 (x0, x1, x2, x3) in two words -> fp16 pairs (x0, x2), (x1, x3).
__device__ __forceinline__ uint2 x4_to_fp16_permuted(uint32_t w01, uint32_t w23) {
    const float f0 = __uint_as_float(w01 << 16), f1 = __uint_as_float(w01 & 0xFFFF0000u);
    const float f2 = __uint_as_float(w23 << 16), f3 = __uint_as_float(w23 & 0xFFFF0000u);
    __half2 a = __floats2half2_rn(f0, f2), b = __floats2half2_rn(f1, f3);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t *>(&a);
    o.y = *reinterpret_cast<uint32_t *>(&b);
    return o;
}

// bf16 (x0..x7) -> fp16 pairs (x0,x2) (x1,x3) (x4,x6) (x5,x7).
__device__ __forceinline__ uint4 x8_to_fp16_permuted(uint4 v) {
    const uint2 lo = x4_to_fp16_permuted(v.x, v.y), hi = x4_to_fp16_permuted(v.z, v.w);
    return make_uint4(lo.x, lo.y, hi.x, hi.y);
}

// Nonzero if any of the 8 bf16 values of v is finite and too large for fp16:
// |x| >= 65536 (its fp16 conversion overflows to inf).  Per 16-bit half, with
// a = |x| bits: 0x4780 = 65536 <= a < 0x7F80 = inf, i.e. a - 0x4780 < 0x3800.
// (Values below the fp16 normal range are not flagged: bf16 values down to
// 2^-17 convert exactly, and a smaller one is off by at most 2^-25, which
// moves a product by at most 2^-25 |w|.)
__device__ __forceinline__ uint32_t x8_fp16_range_bad(uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t bad = 0;
    #pragma unroll
    for (int i = 0; i < 4; ++i) bad |= __vcmpltu2(__vsub2(w[i] & 0x7FFF7FFFu, 0x47804780u), 0x38003800u);
    return bad;
}

// Nonzero if an fp16 scale, given as its bit pattern, is finite and so large
// that (q - 8) * d overflows fp16 for q = 0: 8188 < |d| < inf.
__device__ __forceinline__ bool scale_fp16_range_bad(uint32_t dbits) {
    const uint32_t a = dbits & 0x7FFFu;
    return a >= 0x7000u && a < 0x7C00u;
}

// The slow path of the scale check, run only where a fast path produced a
// non-finite sum: scan the scales of weight rows [n0, n1) of a Q4_0 matrix
// with K weights per row and flag Q4_DEVERR_FP16_RANGE if one is out of range.
static __device__ __noinline__ void scan_scales_fp16_range(const uint8_t *W, int64_t n0, int64_t n1, int64_t N, int64_t K,
                                                    unsigned *err) {
    const int64_t row_bytes = K / 32 * 18;
    for (int64_t n = n0; n < n1 && n < N; ++n)
        for (int64_t b = 0; b < K / 32; ++b) {
            const uint8_t *p = W + n * row_bytes + 18 * b;
            if (scale_fp16_range_bad(static_cast<uint32_t>(p[0]) | (static_cast<uint32_t>(p[1]) << 8))) {
                atomicOr(err, (unsigned)Q4_DEVERR_FP16_RANGE);
                return;
            }
        }
}

}  // namespace q4dev
