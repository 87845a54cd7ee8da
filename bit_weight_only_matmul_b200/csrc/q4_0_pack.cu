// q4_0_pack.cu -- Q4_0 packing, standalone dequantization and the portable
// GEMM kernel (any K % 32 == 0, any M; also the fallback for shapes the fast
// kernels do not take).
//
// Q4_0 block (GGUF convention; the pages name "Q4_0 GGUF" weights:
// voxtral-mini-realtime-rs (Shannon-Prime fork) README, "RTF Benchmark
// Results"): 18 bytes = fp16 scale d, then qs[16]; qs[j] holds code j in its
// low nibble and code j+16 in its high nibble; w = (q - 8) * d.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "q4_0_internal.cuh"

namespace {

constexpr int kBlockBytes = 18;

// One thread per Q4_0 block.
__global__ void pack_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ scales,
                            uint8_t *__restrict__ W, int64_t nblocks, int64_t K) {
    const int64_t nb_row = K / 32;
    for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks;
         b += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = b / nb_row, kb = b % nb_row;
        const uint4 *src = reinterpret_cast<const uint4 *>(codes + n * K + kb * 32);
        const uint4 lo = __ldg(src), hi = __ldg(src + 1);   // codes 0..15, 16..31
        const uint32_t l[4] = {lo.x, lo.y, lo.z, lo.w};
        const uint32_t h[4] = {hi.x, hi.y, hi.z, hi.w};
        uint16_t *dst = reinterpret_cast<uint16_t *>(W + b * kBlockBytes);   // 2-byte aligned
        dst[0] = scales[b];
        #pragma unroll
        for (int w = 0; w < 4; ++w) {
            // qs byte j = (code j & 15) | (code j+16 & 15) << 4, for the 4 bytes of word w
            const uint32_t q = (l[w] & 0x0F0F0F0Fu) | ((h[w] & 0x0F0F0F0Fu) << 4);
            dst[1 + 2 * w] = static_cast<uint16_t>(q & 0xFFFFu);
            dst[2 + 2 * w] = static_cast<uint16_t>(q >> 16);
        }
    }
}

// One thread per Q4_0 block: 32 exact fp32 weights.
__global__ void dequant_kernel(const uint8_t *__restrict__ W, float *__restrict__ out, int64_t nblocks) {
    for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks;
         b += (int64_t)gridDim.x * blockDim.x) {
        const uint16_t *src = reinterpret_cast<const uint16_t *>(W + b * kBlockBytes);
        const float d = __half2float(__ushort_as_half(src[0]));
        float w[32];
        #pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t two = src[1 + j];   // qs bytes 2j, 2j+1
            w[2 * j] = static_cast<float>(static_cast<int>(two & 0xF) - 8) * d;
            w[2 * j + 16] = static_cast<float>(static_cast<int>((two >> 4) & 0xF) - 8) * d;
            w[2 * j + 1] = static_cast<float>(static_cast<int>((two >> 8) & 0xF) - 8) * d;
            w[2 * j + 17] = static_cast<float>(static_cast<int>((two >> 12) & 0xF) - 8) * d;
        }
        float4 *dst = reinterpret_cast<float4 *>(out + b * 32);   // row n*K + 32*kb, 16-byte aligned
        #pragma unroll
        for (int j = 0; j < 8; ++j) dst[j] = make_float4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
    }
}

// Row-interleaved gate/up weight for the fused SwiGLU epilogue: destination
// rows 128i .. 128i+63 are gate rows 64i .. 64i+63, rows 128i+64 .. 128i+127
// the up rows of the same features.  One warp per destination row, 16-byte
// copies (rows of K/32*18 bytes, a multiple of 16 when K % 256 == 0).
__global__ void interleave_kernel(const uint8_t *__restrict__ Wg, const uint8_t *__restrict__ Wu,
                                  uint8_t *__restrict__ Wgu, int64_t F, int64_t row_vec) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t r = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; r < 2 * F; r += warps) {
        const int64_t i = r >> 7, w = r & 127;
        const uint8_t *src = w < 64 ? Wg + (64 * i + w) * row_vec * 16 : Wu + (64 * i + w - 64) * row_vec * 16;
        const uint4 *sv = reinterpret_cast<const uint4 *>(src);
        uint4 *dv = reinterpret_cast<uint4 *>(Wgu + r * row_vec * 16);
        for (int64_t c = lane; c < row_vec; c += 32) dv[c] = sv[c];
    }
}

// Self-test of the failure detection: thread 0 waits on an mbarrier that no
// one arrives on.  The bounded wait must give up after limit_ns, set
// Q4_DEVERR_WAIT_TIMEOUT in the device error word and let the kernel return;
// no copy or MMA is in flight, so nothing else needs to land first.
__global__ void selftest_wait_kernel(unsigned *err, unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        q4dev::mbar_init(&bar, 1);
        q4dev::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)q4dev::mbar_wait(&bar, 0, err, limit_ns);
}

// Portable GEMM: one warp per (row n, chunk of up to 8 rows of X).  Lanes
// stride over the blocks of the row, each block's 32 products are summed in
// fp32 and scaled by d once, and the lanes' partial sums are combined with
// __shfl_xor_sync.
constexpr int kGenericMChunk = 8;

__global__ void generic_kernel(const uint8_t *__restrict__ W, const uint16_t *__restrict__ X,
                               float *__restrict__ Y, int64_t M, int64_t N, int64_t K) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    const int64_t nb_row = K / 32;
    const int64_t mchunks = (M + kGenericMChunk - 1) / kGenericMChunk;
    for (int64_t job = blockIdx.x * (int64_t)(blockDim.x / 32) + threadIdx.x / 32; job < N * mchunks;
         job += warps) {
        const int64_t n = job / mchunks;
        const int64_t m0 = (job % mchunks) * kGenericMChunk;
        const int mc = static_cast<int>((M - m0) < kGenericMChunk ? (M - m0) : kGenericMChunk);
        float acc[kGenericMChunk];
        #pragma unroll
        for (int i = 0; i < kGenericMChunk; ++i) acc[i] = 0.f;
        for (int64_t kb = lane; kb < nb_row; kb += 32) {
            const uint16_t *blk = reinterpret_cast<const uint16_t *>(W + (n * nb_row + kb) * kBlockBytes);
            const float d = __half2float(__ushort_as_half(__ldg(blk)));
            float q[32];
            #pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t two = __ldg(blk + 1 + j);
                q[2 * j] = static_cast<float>(static_cast<int>(two & 0xF) - 8);
                q[2 * j + 16] = static_cast<float>(static_cast<int>((two >> 4) & 0xF) - 8);
                q[2 * j + 1] = static_cast<float>(static_cast<int>((two >> 8) & 0xF) - 8);
                q[2 * j + 17] = static_cast<float>(static_cast<int>((two >> 12) & 0xF) - 8);
            }
            #pragma unroll
            for (int i = 0; i < kGenericMChunk; ++i) {
                if (i < mc) {
                    const uint4 *xr = reinterpret_cast<const uint4 *>(X + (m0 + i) * K + kb * 32);
                    float s = 0.f;
                    #pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const uint4 x8 = __ldg(xr + v);
                        const uint32_t xw[4] = {x8.x, x8.y, x8.z, x8.w};
                        #pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            s = fmaf(__uint_as_float(xw[e] << 16), q[8 * v + 2 * e], s);
                            s = fmaf(__uint_as_float(xw[e] & 0xFFFF0000u), q[8 * v + 2 * e + 1], s);
                        }
                    }
                    acc[i] = fmaf(d, s, acc[i]);
                }
            }
        }
        #pragma unroll
        for (int i = 0; i < kGenericMChunk; ++i) {
            float v = acc[i];
            #pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && i < mc) Y[(m0 + i) * N + n] = v;
        }
    }
}

int grid_for(int64_t work, int threads) {
    const int64_t g = (work + threads - 1) / threads;
    return static_cast<int>(g < 1 ? 1 : (g > 65535 * 8 ? 65535 * 8 : g));
}

}  // namespace

namespace q4 {

cudaError_t launch_pack(const uint8_t *codes, const uint16_t *scales, uint8_t *W, int64_t N, int64_t K,
                        cudaStream_t s) {
    const int64_t nblocks = N * (K / 32);
    pack_kernel<<<grid_for(nblocks, 256), 256, 0, s>>>(codes, scales, W, nblocks, K);
    return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t *W, float *out, int64_t N, int64_t K, cudaStream_t s) {
    const int64_t nblocks = N * (K / 32);
    dequant_kernel<<<grid_for(nblocks, 256), 256, 0, s>>>(W, out, nblocks);
    return cudaGetLastError();
}

cudaError_t launch_interleave_gate_up(const uint8_t *Wg, const uint8_t *Wu, uint8_t *Wgu, int64_t F, int64_t K,
                                     cudaStream_t s) {
    const int64_t rows = 2 * F;
    interleave_kernel<<<grid_for(rows * 32, 256), 256, 0, s>>>(Wg, Wu, Wgu, F, K / 32 * 18 / 16);
    return cudaGetLastError();
}

cudaError_t launch_selftest_wait(const DeviceInfo &dev, unsigned long long limit_ns, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(dev.err, limit_ns);
    return cudaGetLastError();
}

cudaError_t launch_zero(float *Y, int64_t count, cudaStream_t s) {
    return cudaMemsetAsync(Y, 0, static_cast<size_t>(count) * sizeof(float), s);
}

cudaError_t launch_generic(const Problem *probs, int count, const DeviceInfo &dev, cudaStream_t s) {
    for (int i = 0; i < count; ++i) {
        const Problem &p = probs[i];
        const int64_t jobs = p.N * ((p.M + kGenericMChunk - 1) / kGenericMChunk);
        const int64_t ctas = (jobs + 7) / 8;
        const int64_t cap = static_cast<int64_t>(dev.sm_count) * 16;
        generic_kernel<<<static_cast<int>(ctas < cap ? ctas : cap), 256, 0, s>>>(p.W, p.X, p.Y, p.M, p.N, p.K);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace q4
