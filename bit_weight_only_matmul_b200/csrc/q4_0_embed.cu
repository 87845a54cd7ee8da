// q4_0_embed.cu -- two memory-bound utilities around the product: the Q4_0
// row gather (an embedding lookup that dequantizes only the rows it needs)
// and the quantization of float32 weights to Q4_0 blocks.
//
// Gather: the pages keep the 131072 x 3072 token-embedding table in Q4 and
// dequantize the looked-up rows on the CPU, where the fp32 table (1.5 GiB)
// would not fit their budget (hakusoku.com story 5135, linear ops and
// embeddings; voxtral-mini-realtime-rs (Shannon-Prime fork) README, "WASM
// Constraints Solved", item 3).  Here a warp writes 512 contiguous bytes of
// the fp32 output per step: four blocks of a row, lane (b, c) the four
// weights of chunk c of block b (chunks 0-3 the low nibbles of qs bytes
// 4c..4c+3, chunks 4-7 the high nibbles of bytes 4(c-4)..), one 16-byte
// store per lane.  Each weight (q - 8) * d is exact in fp32.  An id outside
// [0, V) writes a zero row and sets Q4_DEVERR_BAD_INDEX.
//
// Quantize: the GGUF Q4_0 rule the pages apply offline (their
// quantize_tts_gguf.py, named in the voxtral-mini-realtime-rs README, TTS
// section), four blocks per warp step (a float4 per lane): the value of
// largest magnitude (the first on ties) over each block's eight lanes by a
// shuffle reduction, d = m / -8, id = 1/d (0 if d == 0),
// q = min(15, trunc(x * id + 8.5)) with the product and the sum rounded
// separately (no fused multiply-add), fp16(d) rounded to nearest even.
#include <cuda_fp16.h>

#include "q4_0_internal.cuh"

namespace {

constexpr int kBlockBytes = 18;


__global__ void gather_kernel(const uint8_t *__restrict__ W, const int32_t *__restrict__ ids,
                              float *__restrict__ out, int64_t T, int64_t V, int64_t nb, unsigned *err) {
    const int lane = threadIdx.x & 31;
    const int64_t quads = (nb + 3) / 4;   // warp units per row
    const int64_t units = T * quads;
    const int64_t warp0 = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int bsub = lane >> 3, c = lane & 7, cc = c & 3, sh = c < 4 ? 0 : 4;
    for (int64_t u = warp0; u < units; u += warps) {
        const int64_t t = u / quads;
        const int64_t b = (u - t * quads) * 4 + bsub;
        if (b >= nb) continue;
        const int64_t v = ids[t];
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        if (v >= 0 && v < V) {
            const uint16_t *blk = reinterpret_cast<const uint16_t *>(W + (v * nb + b) * kBlockBytes);
            const float d = __half2float(__ushort_as_half(blk[0]));
            const uint32_t qs = static_cast<uint32_t>(blk[1 + 2 * cc]) | (static_cast<uint32_t>(blk[2 + 2 * cc]) << 16);
            o.x = static_cast<float>(static_cast<int>((qs >> sh) & 0xF) - 8) * d;
            o.y = static_cast<float>(static_cast<int>((qs >> (8 + sh)) & 0xF) - 8) * d;
            o.z = static_cast<float>(static_cast<int>((qs >> (16 + sh)) & 0xF) - 8) * d;
            o.w = static_cast<float>(static_cast<int>((qs >> (24 + sh)) & 0xF) - 8) * d;
        } else if (b == 0 && c == 0) {
            atomicOr(err, (unsigned)Q4_DEVERR_BAD_INDEX);
        }
        // weights 4cc..4cc+3 of the low (c < 4) or high (c >= 4) half of block b; a
        // streaming store: the rows are read by the next kernel, not by this one
        __stcs(reinterpret_cast<float4 *>(out + t * nb * 32 + b * 32) + c, o);
    }
}

__global__ void quantize_kernel(const float *__restrict__ X, uint8_t *__restrict__ W, int64_t nblocks) {
    // a warp takes four blocks per step: lane (b, c) holds values 4c..4c+3 of block b
    const int lane = threadIdx.x & 31, c = lane & 7;
    const int64_t warp0 = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t quads = (nblocks + 3) / 4;
    for (int64_t qd = warp0; qd < quads; qd += warps) {
        const int64_t b = qd * 4 + (lane >> 3);
        const bool live = b < nblocks;
        const float4 v = live ? reinterpret_cast<const float4 *>(X + b * 32)[c] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float x[4] = {v.x, v.y, v.z, v.w};
        // the first of the largest magnitudes: in the lane, then over the block's 8 lanes
        float a = fabsf(x[0]), m = x[0];
        int at = 4 * c;
        #pragma unroll
        for (int i = 1; i < 4; ++i) {
            const float ai = fabsf(x[i]);
            if (ai > a) { a = ai; m = x[i]; at = 4 * c + i; }
        }
        #pragma unroll
        for (int off = 4; off > 0; off >>= 1) {
            const float a2 = __shfl_xor_sync(0xffffffffu, a, off);
            const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
            const int at2 = __shfl_xor_sync(0xffffffffu, at, off);
            if (a2 > a || (a2 == a && at2 < at)) { a = a2; m = m2; at = at2; }
        }
        if (a == 0.0f) m = 0.0f;   // an all-zero block (of either sign) has m = +0
        const float d = __fdiv_rn(m, -8.0f);
        const float id = d != 0.0f ? __frcp_rn(d) : 0.0f;
        uint32_t qw = 0;   // this lane's four codes, one per byte
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
            int q = __float2int_rz(__fadd_rn(__fmul_rn(x[i], id), 8.5f));
            q = q > 15 ? 15 : q;
            qw |= static_cast<uint32_t>(q) << (8 * i);
        }
        // lane c < 4 holds codes 4c..4c+3 (low nibbles of qs bytes 4c..4c+3), lane c+4
        // the codes 16+4c.. that go in the high nibbles of the same bytes
        const uint32_t hiw = __shfl_down_sync(0xffffffffu, qw, 4);
        if (live && c < 4) {
            const uint32_t bytes = qw | (hiw << 4);
            uint16_t *blk = reinterpret_cast<uint16_t *>(W + b * kBlockBytes);
            blk[1 + 2 * c] = static_cast<uint16_t>(bytes & 0xFFFFu);
            blk[2 + 2 * c] = static_cast<uint16_t>(bytes >> 16);
            if (c == 0) blk[0] = __half_as_ushort(__float2half_rn(d));
        }
    }
}

int grid_for(int64_t warps_needed, int sm_count) {
    const int64_t ctas = (warps_needed + 7) / 8;
    const int64_t cap = static_cast<int64_t>(sm_count) * 16;
    return static_cast<int>(ctas < 1 ? 1 : (ctas < cap ? ctas : cap));
}

}  // namespace

namespace q4 {

cudaError_t launch_gather(const uint8_t *W, const int32_t *ids, float *out, int64_t T, int64_t V, int64_t D,
                          const DeviceInfo &dev, cudaStream_t s) {
    const int64_t nb = D / 32;
    gather_kernel<<<grid_for(T * ((nb + 3) / 4), dev.sm_count), 256, 0, s>>>(W, ids, out, T, V, nb, dev.err);
    return cudaGetLastError();
}

cudaError_t launch_quantize(const float *X, uint8_t *W, int64_t N, int64_t K, const DeviceInfo &dev,
                            cudaStream_t s) {
    const int64_t nblocks = N * (K / 32);
    quantize_kernel<<<grid_for((nblocks + 3) / 4, dev.sm_count), 256, 0, s>>>(X, W, nblocks);
    return cudaGetLastError();
}

}  // namespace q4
