// q4_0_decode_tmem.cu -- the memory-bound decode path (M <= 32) on the
// 5th-generation tensor cores: one persistent launch streams the Q4_0 weights
// of one or many problems once from HBM; worker warps dequantize them in
// registers into tensor memory, and tcgen05.mma multiplies them with the
// (few) activation rows.
//
// The pages' token loop runs a Q4 matmul for every decoder linear of each of
// the 26 layers (voxtral-mini-realtime-rs (Shannon-Prime fork) README,
// "Architecture Summary"; decode is most of the time: "Pipeline Overlap"),
// with batch-2 CFG and fused QKV / gate-up projections ("TTS
// (Text-to-Speech)", optimizations), and up to 32 concurrent sequences in the
// Tenstorrent port (Voxtral-Mini-4B-Realtime-2602-tt-p300x2 README, serving).
//
// Why tensor memory: at ~6.5 TB/s a B200 must consume ~1.2e13 weights/s, about
// 3 issue slots per weight at the highest clock; dequantizing into registers
// and reducing with FMAs, shuffles or mma.sync costs 2.5-3.2 instructions per
// weight (measured).  Here a weight costs ~1.6 (a mask-or, a subtract and a
// multiply per pair of weights) and the products and sums run on tcgen05.
//
// Per CTA (one per SM): a producer warp, an MMA warp, an X warp, 8 worker
// warps and 4 epilogue warps.
//  * item = 128 weight rows x all of K of one problem; items are sorted by K
//    (largest first) on the host and dealt to the CTAs in boustrophedon order;
//  * stage = 256 k of the item (8 Q4_0 blocks, 144 contiguous bytes per row)
//    plus the same 256 k of every row of X, in a ring: the weights as one TMA
//    box (128 rows x 144 bytes), the X rows as 1-D bulk copies;
//  * worker warp (quadrant q, half h) owns tensor-memory lanes 32q..32q+31 =
//    weight rows and blocks 4h..4h+3 of each stage: it turns codes and scale
//    into fp16 w = (q - 8) * d (one rounding) and writes them with tcgen05.st
//    as the MMA's A operand (three buffers);
//  * the X warp converts the stage's X rows to fp16 into the 128-byte-swizzled
//    B operand (three buffers);
//  * the MMA thread issues 16 tcgen05.mma (kind::f16, M=128, N=NN, K=16) per
//    stage into the item's accumulator (two accumulators alternate between
//    items), and releases A/B with tcgen05.commit;
//  * the epilogue warps read an item's accumulator (tcgen05.ld) and store
//    Y[m, n] for its 128 rows n (one coalesced run per m).
// Inside each 32-k block the k order is permuted identically for both
// operands (positions 1 and 2 of every 4 swapped), so that the nibble pairs
// are used in the order the packed bytes hold them.
// Numerics: each weight is rounded once to fp16 (relative error <= 2^-11,
// inside the 1e-3 tolerance of the method) and X is exact in fp16 within its
// normal range; products are exact and accumulation is fp32.  Operands beyond
// the fp16 range (|x| > 65504, |d| > 8188) overflow to +-inf.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <vector>

#include "q4_0_internal.cuh"
#include "q4_0_convert.cuh"
#include "q4_0_tcgen05.cuh"
#include "q4_0_tmap.cuh"

namespace {

using namespace q4dev;

constexpr int kRows = 128;                  // weight rows per item = tensor-memory lanes
constexpr int kStageK = 256;                // k per stage: 8 Q4_0 blocks
constexpr int kRawRow = 144;                // bytes of one row per stage
constexpr int kRawW = kRows * kRawRow;      // 18432
constexpr int kXRow = kStageK * 2;          // 512 bytes of one X row per stage
constexpr int kABufs = 3;                   // A and B operand buffers
constexpr int kWarpProd = 0, kWarpMMA = 1, kWarpX = 2, kWarp0 = 3, kWorkers = 8, kWarpEpi0 = 11, kNumEpi = 4;
constexpr int kThreads = 32 * (kWarpEpi0 + kNumEpi);   // 480
constexpr uint32_t kTmemCols = 512;
constexpr int kACol = 0;                    // A: 3 buffers x 128 columns (256 fp16 per row)
constexpr int kDCol = 384;                  // D: 2 accumulators x NN columns

// NN = MMA N (16 or 32 activation rows)
template <int NN> constexpr int raw_bytes() { return kRawW + NN * kXRow; }
template <int NN> constexpr int ring() { return NN == 16 ? 6 : 4; }
template <int NN> constexpr int b_bytes() { return NN * kStageK * 2; }   // 4 swizzle atoms of NN rows x 128 B

struct TProblem {
    const uint8_t *W;
    const uint16_t *X;
    float *Y;
    int M, N, K;
    int stages;        // K / 256
    int item_begin;    // first item index of this problem
};

// CAP problems per launch (the tensor maps live in the kernel parameters).
template <int CAP>
struct alignas(64) TParams {
    CUtensorMap wmap[CAP];   // Q4_0 bytes [N, K/32*18], box 144 x 128
    int count;
    int total_items;
    unsigned *err;
    TProblem p[CAP];
};

template <int NN>
struct Smem {
    uint8_t raw[ring<NN>()][raw_bytes<NN>()];  // W rows (pitch 144) then X rows (pitch 512)
    uint8_t b[kABufs][b_bytes<NN>()];          // B operand, 1024-byte aligned
    uint64_t raw_full[ring<NN>()], raw_empty[ring<NN>()];
    uint64_t a_full[kABufs], b_full[kABufs], ab_empty[kABufs];
    uint64_t d_full[2], d_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
};

template <class TP>
__device__ __forceinline__ int find_problem(const TP &P, int item) {
    int lo = 0, hi = P.count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.p[mid].item_begin <= item) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// One CTA's sequence of (item, stage).
struct Seq {
    int round, item, prob, row0, stage, nstages;
    uint32_t nitems;   // items this CTA finished before the current one
    template <class TP>
    __device__ __forceinline__ void load(const TP &P) {
        const int G = gridDim.x;
        const int pos = (round & 1) ? (G - 1 - static_cast<int>(blockIdx.x)) : static_cast<int>(blockIdx.x);
        item = round * G + pos;
        if (item >= P.total_items) { item = -1; return; }
        prob = find_problem(P, item);
        row0 = (item - P.p[prob].item_begin) * kRows;
        stage = 0;
        nstages = P.p[prob].stages;
    }
    template <class TP>
    __device__ __forceinline__ void start(const TP &P) { round = 0; nitems = 0; load(P); }
    template <class TP>
    __device__ __forceinline__ void next(const TP &P) {
        if (++stage < nstages) return;
        ++round;
        ++nitems;
        load(P);
    }
};

template <class S>
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, S &sm, unsigned *err) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait_suspend(bar, parity)) {
        if (*reinterpret_cast<volatile int *>(&sm.abort_flag)) return false;
        if (global_ns() - t0 > kWaitLimitNs) {
            atomicOr(err, (unsigned)Q4_DEVERR_WAIT_TIMEOUT);
            *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
            return false;
        }
    }
    return true;
}

// Blocks 4*HALF .. 4*HALF+3 of a stage row, held in w[] = bytes
// [64*HALF, 64*HALF + 80) of the 144-byte row: 64 tensor-memory columns (16
// per block, fp16 pairs in the permuted k order above).  Blocks at an even
// index start 4-byte aligned in w[], odd ones at 2 mod 4.
template <int HALF>
__device__ __forceinline__ void dequant_half(const uint32_t (&w)[20], uint32_t (&cols)[64]) {
    #pragma unroll
    for (int jb = 0; jb < 4; ++jb) {
        const int b = 18 * (4 * HALF + jb) - 64 * HALF;   // byte offset of the block in w[]
        const int wi = b >> 2;
        uint32_t d2, qw[4];
        if ((jb & 1) == 0) {
            d2 = prmt(w[wi], w[wi], 0x1010u);              // (d, d)
            #pragma unroll
            for (int k = 0; k < 4; ++k) qw[k] = prmt(w[wi + k], w[wi + k + 1], 0x5432u);
        } else {
            d2 = prmt(w[wi], w[wi], 0x3232u);
            #pragma unroll
            for (int k = 0; k < 4; ++k) qw[k] = w[wi + 1 + k];
        }
        #pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint32_t c[4];
            q4_word_to_fp16(qw[k], d2, c);
            cols[16 * jb + 2 * k] = c[0];
            cols[16 * jb + 2 * k + 1] = c[1];
            cols[16 * jb + 8 + 2 * k] = c[2];
            cols[16 * jb + 8 + 2 * k + 1] = c[3];
        }
    }
}

template <int NN, int CAP>
__global__ void __launch_bounds__(kThreads, 1) decode_tmem_kernel(const __grid_constant__ TParams<CAP> P) {
    constexpr int RS = ring<NN>();
    constexpr uint32_t kIdesc = f16_idesc(128, NN, false);
    extern __shared__ uint8_t smem_raw[];
    using SM = Smem<NN>;
    SM &S = *reinterpret_cast<SM *>(align_smem<1024>(smem_raw));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < RS; ++s) {
            mbar_init(&S.raw_full[s], 1);
            mbar_init(&S.raw_empty[s], kWorkers + 1);
        }
        for (int s = 0; s < kABufs; ++s) {
            mbar_init(&S.a_full[s], kWorkers);
            mbar_init(&S.b_full[s], 1);
            mbar_init(&S.ab_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&S.d_full[s], 1);
            mbar_init(&S.d_empty[s], kNumEpi);
        }
        mbar_init(&S.mma_done, 1);
        S.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMMA) tmem_alloc(&S.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    uint32_t prod_issued = 0;   // stages whose copies the producer issued

    if (warp == kWarpProd) {
        // ---------------------------------------------------------------- loads
        Seq q{};
        q.start(P);
        for (; q.item >= 0; q.next(P)) {
            const TProblem &pr = P.p[q.prob];
            const uint32_t g = prod_issued;
            const int slot = g % RS;
            bool ok = true;
            if (lane == 0) ok = wait_or_abort(&S.raw_empty[slot], ((g / RS) & 1) ^ 1, S, P.err);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            // weights: one TMA box (rows past N are zero-filled and still counted)
            if (lane == 0) {
                mbar_arrive_expect_tx(&S.raw_full[slot], kRawW + pr.M * kXRow);
                tma_load_2d(S.raw[slot], &P.wmap[q.prob], q.stage * kRawRow, q.row0, &S.raw_full[slot]);
            }
            __syncwarp();
            for (int m = lane; m < pr.M; m += 32)
                bulk_g2s(S.raw[slot] + kRawW + m * kXRow,
                         pr.X + static_cast<int64_t>(m) * pr.K + static_cast<int64_t>(q.stage) * kStageK, kXRow,
                         &S.raw_full[slot]);
            ++prod_issued;
        }
    } else if (warp == kWarpMMA) {
        // ---------------------------------------------------------------- MMA issue
        if (lane == 0) {
            uint32_t g = 0;
            Seq q{};
            q.start(P);
            for (; q.item >= 0; q.next(P), ++g) {
                const int buf = g % kABufs;
                const uint32_t par = (g / kABufs) & 1;
                const uint32_t ib = q.nitems & 1;   // accumulator of this item
                if (q.stage == 0 && !wait_or_abort(&S.d_empty[ib], ((q.nitems >> 1) & 1) ^ 1, S, P.err)) break;
                if (!wait_or_abort(&S.a_full[buf], par, S, P.err)) break;
                if (!wait_or_abort(&S.b_full[buf], par, S, P.err)) break;
                tc_fence_after();
                const uint64_t bdesc = sw128_kmajor_desc(smem_addr(S.b[buf]));
                #pragma unroll
                for (int i = 0; i < 8; ++i)
                    #pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        // block i = k [32i, 32i+32): swizzle atom i/2, byte offset 64*(i%2) + 32*j in its rows
                        const uint32_t off = (i >> 1) * (NN * 128) + (i & 1) * 64 + j * 32;
                        tc_mma_ts(tmem + kDCol + NN * ib, tmem + kACol + 128 * buf + 16 * i + 8 * j,
                                  bdesc + (off >> 4), kIdesc, (q.stage | i | j) != 0);
                    }
                tc_commit(&S.ab_empty[buf]);
                if (q.stage == q.nstages - 1) tc_commit(&S.d_full[ib]);
            }
            tc_commit(&S.mma_done);
            if (!wait_or_abort(&S.mma_done, 0, S, P.err)) mbar_wait(&S.mma_done, 0, P.err);
        }
    } else if (warp == kWarpX) {
        // ---------------------------------------------------------------- X rows -> B operand (fp16)
        uint32_t g = 0;
        Seq q{};
        q.start(P);
        for (; q.item >= 0; q.next(P), ++g) {
            const TProblem &pr = P.p[q.prob];
            const int slot = g % RS, buf = g % kABufs;
            bool ok = true;
            if (lane == 0) {
                ok = wait_or_abort(&S.raw_full[slot], (g / RS) & 1, S, P.err);
                if (ok) ok = wait_or_abort(&S.ab_empty[buf], ((g / kABufs) & 1) ^ 1, S, P.err);
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            // 128-byte swizzle: atom = 64 k x NN rows (NN*128 bytes), 8-row groups of 1024 bytes
            for (int c = lane; c < pr.M * 32; c += 32) {
                const int m = c >> 5, kc = c & 31;
                const uint4 v = *reinterpret_cast<const uint4 *>(S.raw[slot] + kRawW + m * kXRow + kc * 16);
                *reinterpret_cast<uint4 *>(S.b[buf] + (kc >> 3) * (NN * 128) + (m >> 3) * 1024 + (m & 7) * 128 +
                                           (((kc & 7) ^ (m & 7)) * 16)) = x8_to_fp16_permuted(v);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&S.b_full[buf]);
                mbar_arrive(&S.raw_empty[slot]);
            }
        }
    } else if (warp >= kWarp0 && warp < kWarp0 + kWorkers) {
        // ---------------------------------------------------------------- weights -> A operand (fp16)
        const int quad = warp & 3;               // tensor-memory lanes 32*quad ..
        const int half = (warp - kWarp0) >> 2;   // blocks 4*half .. 4*half+3 of each stage
        const uint32_t lane_base = uint32_t(32 * quad) << 16;
        uint32_t g = 0;
        Seq q{};
        q.start(P);
        for (; q.item >= 0; q.next(P), ++g) {
            const int slot = g % RS, buf = g % kABufs;
            if (!wait_or_abort(&S.raw_full[slot], (g / RS) & 1, S, P.err)) break;
            // this thread's half row: bytes [64*half, 64*half + 80) of the 144-byte stage row
            uint32_t w[20];
            {
                const uint4 *src =
                    reinterpret_cast<const uint4 *>(S.raw[slot] + (32 * quad + lane) * kRawRow + 64 * half);
                #pragma unroll
                for (int i = 0; i < 5; ++i) {
                    const uint4 v = src[i];
                    w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
                }
            }
            fence_proxy_async_smem();   // the producer's next copies may land in this slot
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.raw_empty[slot]);
            uint32_t cols[64];
            if (half == 0) dequant_half<0>(w, cols);
            else dequant_half<1>(w, cols);
            // A[buf] was last read by the MMAs of stage g-3
            if (!wait_or_abort(&S.ab_empty[buf], ((g / kABufs) & 1) ^ 1, S, P.err)) break;
            tc_fence_after();
            {
                const uint32_t ta = tmem + lane_base + kACol + 128 * buf + 64 * half;
                uint32_t lo[32], hi[32];
                #pragma unroll
                for (int i = 0; i < 32; ++i) { lo[i] = cols[i]; hi[i] = cols[32 + i]; }
                tc_st_32(ta, lo);
                tc_st_32(ta + 32, hi);
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.a_full[buf]);
        }
    } else {
        // ---------------------------------------------------------------- epilogue: accumulator -> Y
        const int quad = warp & 3;
        const uint32_t lane_base = uint32_t(32 * quad) << 16;
        Seq q{};
        q.start(P);
        for (uint32_t it = 0; q.item >= 0; ++it) {
            const TProblem &pr = P.p[q.prob];
            const int row0 = q.row0;
            const uint32_t ib = it & 1;
            if (!wait_or_abort(&S.d_full[ib], (it >> 1) & 1, S, P.err)) break;
            tc_fence_after();
            float v[NN];
            tc_ld_cols<NN>(tmem + lane_base + kDCol + NN * ib, v);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.d_empty[ib]);
            const int n = row0 + 32 * quad + lane;
            if (n < pr.N) {
                #pragma unroll
                for (int m = 0; m < NN; ++m)
                    if (m < pr.M) pr.Y[static_cast<int64_t>(m) * pr.N + n] = v[m];
            }
            const int nst = q.nstages;   // on to the next item
            for (int s = 0; s < nst; ++s) q.next(P);
        }
    }

    tc_fence_before();
    __syncthreads();
    // Abort path: copies issued but never consumed may still be in flight;
    // let them land (bounded) before the CTA exits.
    if (*reinterpret_cast<volatile int *>(&S.abort_flag) && warp == kWarpProd && lane == 0) {
        for (uint32_t i = 0; i < RS && i < prod_issued; ++i) {
            const uint32_t gg = prod_issued - 1 - i;
            mbar_wait(&S.raw_full[gg % RS], (gg / RS) & 1, P.err);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMMA) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int NN>
constexpr size_t smem_bytes() { return sizeof(Smem<NN>) + 1024; }

template <int NN, int CAP>
cudaError_t launch_nn(TParams<CAP> &P, const q4::DeviceInfo &dev, cudaStream_t s) {
    static q4::DeviceOnce configured;
    cudaError_t e = configured.run(dev.device, [] {
        return cudaFuncSetAttribute(decode_tmem_kernel<NN, CAP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem_bytes<NN>()));
    });
    if (e != cudaSuccess) return e;
    const int grid = std::max(1, std::min(dev.sm_count, P.total_items));
    decode_tmem_kernel<NN, CAP><<<grid, kThreads, smem_bytes<NN>(), s>>>(P);
    return cudaGetLastError();
}

// problems[order[0..count)] sorted by K (largest first), count <= CAP
template <int CAP>
cudaError_t launch_cap(const q4::Problem *probs, const int *order, int count, const q4::DeviceInfo &dev,
                       cudaStream_t s) {
    static thread_local TParams<CAP> P;
    P.count = count;
    P.err = dev.err;
    int items = 0;
    int64_t maxM = 1;
    for (int i = 0; i < count; ++i) {
        const q4::Problem &q = probs[order[i]];
        TProblem &t = P.p[i];
        t.W = q.W;
        t.X = q.X;
        t.Y = q.Y;
        t.M = static_cast<int>(q.M);
        t.N = static_cast<int>(q.N);
        t.K = static_cast<int>(q.K);
        t.stages = static_cast<int>(q.K / kStageK);
        t.item_begin = items;
        items += static_cast<int>((q.N + kRows - 1) / kRows);
        maxM = std::max(maxM, q.M);
        if (!q4::get_tensor_map(&P.wmap[i], q.W, q.N, q.K / 32 * 18, q4::kMapWeights128))
            return cudaErrorInvalidValue;
    }
    P.total_items = items;
    if (maxM <= 16) return launch_nn<16, CAP>(P, dev, s);
    return launch_nn<32, CAP>(P, dev, s);
}

constexpr int kSmallCap = 8, kLargeCap = 128;

}  // namespace

namespace q4 {

bool decode_tmem_supports(const Problem &p) {
    return p.M >= 1 && p.M <= 32 && p.K >= kStageK && p.K % kStageK == 0 && p.N >= 1 && p.N < (1LL << 31) &&
           p.K < (1LL << 31) && (reinterpret_cast<uintptr_t>(p.W) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(p.X) & 15) == 0 && tensor_maps_available();
}

cudaError_t launch_decode_tmem(const Problem *probs, int count, const DeviceInfo &dev, cudaStream_t s) {
    if (count <= 0) return cudaSuccess;
    std::vector<int> order(count);
    for (int i = 0; i < count; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return probs[a].K > probs[b].K; });
    for (int done = 0; done < count;) {
        const int n = std::min(count - done, kLargeCap);
        cudaError_t e = n <= kSmallCap ? launch_cap<kSmallCap>(probs, order.data() + done, n, dev, s)
                                       : launch_cap<kLargeCap>(probs, order.data() + done, n, dev, s);
        if (e != cudaSuccess) return e;
        done += n;
    }
    return cudaSuccess;
}

}  // namespace q4
