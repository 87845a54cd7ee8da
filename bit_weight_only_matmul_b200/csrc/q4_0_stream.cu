// q4_0_stream.cu -- a measurement instrument: read a Q4_0 matrix once with
// the decode kernels' weight stream (TMA boxes of 128 rows x 144 bytes = 256 k
// into a ring of shared-memory slots, one persistent CTA per SM) and do
// nothing with it but XOR its 32-bit words into a checksum.  The rate it
// reaches is the ceiling of that access pattern on this GPU: what the decode
// kernels could stream if their arithmetic were free.  The pages have no
// counterpart.
#include <cuda.h>

#include <algorithm>

#include "q4_0_internal.cuh"
#include "q4_0_sched.cuh"
#include "q4_0_tcgen05.cuh"
#include "q4_0_tmap.cuh"

namespace {

using namespace q4dev;

constexpr int kBox = kItemRows * kStageRowBytes;   // 18432 bytes: one 256-k stage of 128 rows
constexpr int kSlots = 10;                         // ring depth (184 KB)
constexpr int kReaders = 4;                        // warps that XOR the landed boxes
constexpr int kThreads = 32 * (1 + kReaders);

struct alignas(64) StreamParams {
    CUtensorMap wmap;      // Q4_0 bytes [N, K/32*18], box 144 x 128
    uint32_t *checksum;
    unsigned *err;
    int items, stages;     // units: items x stages boxes
};

struct Smem {
    uint8_t slot[kSlots][kBox];
    uint64_t full[kSlots], empty[kSlots];
    int abort_flag;
};

__global__ void __launch_bounds__(kThreads, 1) stream_kernel(const __grid_constant__ StreamParams P) {
    extern __shared__ uint8_t smem_raw[];
    Smem &S = *reinterpret_cast<Smem *>(align_smem<128>(smem_raw));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.empty[s], kReaders);
        }
        S.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // CTA b streams units [begin, end): consecutive units of an item walk
    // along K, then the next item, as the decode kernels do
    const int64_t units = static_cast<int64_t>(P.items) * P.stages;
    const int begin = static_cast<int>(units * blockIdx.x / gridDim.x);
    const int end = static_cast<int>(units * (blockIdx.x + 1) / gridDim.x);
    uint32_t issued = 0;
    if (warp == 0) {
        if (lane == 0) {
            for (int u = begin; u < end; ++u, ++issued) {
                const int s = issued % kSlots;
                if (!wait_or_abort(&S.empty[s], ((issued / kSlots) & 1) ^ 1, &S.abort_flag, P.err)) break;
                mbar_arrive_expect_tx(&S.full[s], kBox);
                tma_load_2d(S.slot[s], &P.wmap, (u % P.stages) * kStageRowBytes, (u / P.stages) * kItemRows,
                            &S.full[s]);
            }
        }
    } else {
        const int r = warp - 1;
        uint32_t x = 0, n = 0;
        for (int u = begin; u < end; ++u, ++n) {
            const int s = n % kSlots;
            if (!wait_or_abort(&S.full[s], (n / kSlots) & 1, &S.abort_flag, P.err)) break;
            // reader r takes every kReaders-th 16-byte chunk of the box
            const uint4 *p = reinterpret_cast<const uint4 *>(S.slot[s]);
            #pragma unroll 4
            for (int i = r * 32 + lane; i < kBox / 16; i += 32 * kReaders) {
                const uint4 v = p[i];
                x ^= v.x ^ v.y ^ v.z ^ v.w;
            }
            fence_proxy_async_smem();   // the next box may land in this slot
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.empty[s]);
        }
        if (x) atomicXor(P.checksum, x);
    }
    __syncthreads();
    // abort path: let issued boxes land (bounded) before the CTA exits
    if (*reinterpret_cast<volatile int *>(&S.abort_flag) && warp == 0 && lane == 0) {
        for (uint32_t i = 0; i < kSlots && i < issued; ++i) {
            const uint32_t g = issued - 1 - i;
            mbar_wait(&S.full[g % kSlots], (g / kSlots) & 1, P.err);
        }
    }
}

constexpr size_t kSmemBytes = sizeof(Smem) + 128;
static_assert(kSmemBytes <= 232448, "shared memory budget");

}  // namespace

namespace q4 {

bool stream_read_supports(int64_t N, int64_t K) {
    return N >= 1 && K >= kStageK && K % kStageK == 0 && N < (1LL << 31) && K < (1LL << 31) &&
           (N + kItemRows - 1) / kItemRows * (K / kStageK) < (1LL << 31) && tensor_maps_available();
}

cudaError_t launch_stream_read(const uint8_t *W, int64_t N, int64_t K, uint32_t *checksum, const DeviceInfo &dev,
                               cudaStream_t s) {
    StreamParams P;
    if (!get_tensor_map(&P.wmap, W, N, K / 32 * 18, kMapWeights128)) return cudaErrorInvalidValue;
    P.checksum = checksum;
    P.err = dev.err;
    P.items = static_cast<int>((N + kItemRows - 1) / kItemRows);
    P.stages = static_cast<int>(K / kStageK);
    static DeviceOnce configured;
    cudaError_t e = configured.run(dev.device, [] {
        return cudaFuncSetAttribute(stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(kSmemBytes));
    });
    if (e != cudaSuccess) return e;
    const int64_t units = static_cast<int64_t>(P.items) * P.stages;
    const int grid = static_cast<int>(std::min<int64_t>(dev.sm_count, units));
    stream_kernel<<<grid, kThreads, kSmemBytes, s>>>(P);
    return cudaGetLastError();
}

}  // namespace q4
