// q4_0_decode_tmem.cu -- the memory-bound decode path for M <= 16 on the
// 5th-generation tensor cores: one persistent launch streams the Q4_0 weights
// of one or many problems once from HBM; worker warps dequantize them in
// registers into tensor memory, and tcgen05.mma multiplies them with the
// (few) activation rows.
//
// The pages' token loop runs a Q4 matmul for every decoder linear of each of
// the 26 layers (voxtral-mini-realtime-rs (Shannon-Prime fork) README,
// "Architecture Summary"; decode is most of the time: "Pipeline Overlap"),
// with batch-2 CFG and fused QKV / gate-up projections ("TTS
// (Text-to-Speech)", optimizations).
//
// Why tensor memory: at ~6.5 TB/s a B200 must consume ~1.2e13 weights/s, about
// 3 issue slots per weight at the highest clock.  Dequantizing into registers
// and reducing with FMAs, shuffles or mma.sync costs 2.5-3.2 instructions per
// weight (measured); here a weight costs ~1.4 (a shift/mask/subtract per
// pair of weights, exact in bf16) and the products and sums run on tcgen05.
//
// Per CTA (one per SM): a producer warp, an MMA warp and 8 worker warps.
//  * item = 128 weight rows x all of K of one problem; items are sorted by K
//    (largest first) on the host and dealt to the CTAs in boustrophedon order;
//  * stage = 256 k of the item (8 Q4_0 blocks, 144 contiguous bytes per row)
//    plus the same 256 k of every row of X, in a 4-deep ring: the weights as
//    one TMA box (128 rows x 144 bytes) per stage, the few X rows as 1-D bulk
//    copies (one issue per byte run costs ~60 cycles per SM, so the weights
//    must not come row by row);
//  * worker warp (quadrant q, half h) owns tensor-memory lanes 32q..32q+31 =
//    weight rows, and blocks 4h..4h+3 of each stage: it turns the 4-bit codes
//    into exact bf16 (q - 8) and writes them to tensor memory (A operand,
//    double-buffered) with tcgen05.st; the workers also copy the stage's X
//    into the 128-byte-swizzled B operand (double-buffered);
//  * the MMA thread multiplies each 32-k block separately (two M=128, N=16,
//    K=16 MMAs into the block's own 16 accumulator columns), so that the
//    workers can apply the block's fp16 scale d exactly in fp32 when they read
//    the partial sums back (tcgen05.ld); the scale never rounds a weight;
//  * at the end of an item the two workers of a quadrant add their partial
//    sums and store Y[m, n] for the 32 rows n of the quadrant (one coalesced
//    128-byte run per m).
// Inside each 32-k block the k order is permuted identically for both
// operands (positions 1 and 2 of every 4 swapped), so that the nibble pairs
// are used in the order the packed bytes hold them.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <vector>

#include "q4_0_internal.cuh"
#include "q4_0_tcgen05.cuh"
#include "q4_0_tmap.cuh"

namespace {

using namespace q4dev;

constexpr int kRows = 128;                  // weight rows per item = tensor-memory lanes
constexpr int kStageK = 256;                // k per stage: 8 Q4_0 blocks
constexpr int kRawRow = 144;                // bytes of one row per stage
constexpr int kRawW = kRows * kRawRow;      // 18432
constexpr int kMaxM = 16;                   // activation rows (the MMA's N)
constexpr int kXRow = kStageK * 2;          // 512 bytes of one X row per stage
constexpr int kRawBytes = kRawW + kMaxM * kXRow;   // 26624
constexpr int kRS = 6;                      // ring depth
constexpr int kBBytes = kMaxM * kStageK * 2;       // 8192: 4 swizzle atoms of 16 rows x 128 bytes
constexpr int kWarpProd = 0, kWarpMMA = 1, kWarpX = 2, kWarp0 = 3, kWorkers = 8;
constexpr int kThreads = 32 * (kWarp0 + kWorkers);  // 352
constexpr uint32_t kTmemCols = 512;
constexpr int kACol = 0;                    // A: 2 buffers x 128 columns (256 bf16 per row)
constexpr int kDCol = 256;                  // D: 2 buffers x (8 blocks x 16 columns)
constexpr uint32_t kIdesc = f16_idesc(128, kMaxM, true);

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

struct Smem {
    uint8_t raw[kRS][kRawBytes];              // W rows (pitch 144) then X rows (pitch 512)
    uint8_t b[2][kBBytes];                    // B operand, 1024-byte aligned
    float comb[2][4][kMaxM][32];              // partial sums handed between the two halves
    uint64_t raw_full[kRS], raw_empty[kRS];
    uint64_t ab_full[2], b_full[2], b_empty[2], d_full[2], d_empty[2];
    uint64_t comb_full[2], comb_empty[2];
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
    __device__ __forceinline__ void start(const TP &P) { round = 0; load(P); }
    template <class TP>
    __device__ __forceinline__ void next(const TP &P) {
        if (++stage < nstages) return;
        ++round;
        load(P);
    }
};

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, Smem &S, unsigned *err) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait_suspend(bar, parity)) {
        if (*reinterpret_cast<volatile int *>(&S.abort_flag)) return false;
        if (global_ns() - t0 > kWaitLimitNs) {
            atomicOr(err, (unsigned)Q4_DEVERR_WAIT_TIMEOUT);
            *reinterpret_cast<volatile int *>(&S.abort_flag) = 1;
            return false;
        }
    }
    return true;
}

// Exact bf16 pairs (q - 8) from one qs word v (bytes 4w..4w+3 of a block):
//   c[0] = elements (4w, 4w+2), c[1] = (4w+1, 4w+3)          (low nibbles)
//   c[2] = elements (4w+16, 4w+18), c[3] = (4w+17, 4w+19)    (high nibbles)
// 0x4300 is bf16 128 (7 fraction bits: 128 + q is exact for q < 16), and
// subtracting bf16 136 leaves q - 8 exactly.
__device__ __forceinline__ void codes_bf16(uint32_t v, uint32_t (&c)[4]) {
    const __nv_bfloat162 off = __halves2bfloat162(__ushort_as_bfloat16(0x4308), __ushort_as_bfloat16(0x4308));
    uint32_t t[4] = {and_or(v, 0x000F000Fu, 0x43004300u), and_or(v >> 8, 0x000F000Fu, 0x43004300u),
                     and_or(v >> 4, 0x000F000Fu, 0x43004300u), and_or(v >> 12, 0x000F000Fu, 0x43004300u)};
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162 *>(&t[i]), off);
        c[i] = *reinterpret_cast<uint32_t *>(&r);
    }
}

// Blocks 4*HALF .. 4*HALF+3 of a stage row, held in w[] = bytes
// [64*HALF, 64*HALF + 80) of the 144-byte row: fp32 scales and 64 tensor-memory
// columns (16 per block, bf16 pairs in the permuted k order above).  Blocks
// at an even index start 4-byte aligned in w[], odd ones at 2 mod 4.
template <int HALF>
__device__ __forceinline__ void dequant_half(const uint32_t (&w)[20], uint32_t (&cols)[64], float (&d)[4]) {
    #pragma unroll
    for (int jb = 0; jb < 4; ++jb) {
        const int b = 18 * (4 * HALF + jb) - 64 * HALF;   // byte offset of the block in w[]
        const int wi = b >> 2;
        uint32_t dbits, qw[4];
        if ((jb & 1) == 0) {
            dbits = w[wi] & 0xFFFFu;
            #pragma unroll
            for (int k = 0; k < 4; ++k) qw[k] = prmt(w[wi + k], w[wi + k + 1], 0x5432u);
        } else {
            dbits = w[wi] >> 16;
            #pragma unroll
            for (int k = 0; k < 4; ++k) qw[k] = w[wi + 1 + k];
        }
        d[jb] = __half2float(__ushort_as_half(static_cast<unsigned short>(dbits)));
        #pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint32_t c[4];
            codes_bf16(qw[k], c);
            cols[16 * jb + 2 * k] = c[0];
            cols[16 * jb + 2 * k + 1] = c[1];
            cols[16 * jb + 8 + 2 * k] = c[2];
            cols[16 * jb + 8 + 2 * k + 1] = c[3];
        }
    }
}

template <int MP, int CAP>
__global__ void __launch_bounds__(kThreads, 1) decode_tmem_kernel(const __grid_constant__ TParams<CAP> P) {
    extern __shared__ uint8_t smem_raw[];
    Smem &S = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRS; ++s) {
            mbar_init(&S.raw_full[s], 1);
            mbar_init(&S.raw_empty[s], kWorkers + 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&S.ab_full[s], kWorkers);
            mbar_init(&S.b_full[s], 1);
            mbar_init(&S.b_empty[s], 1);
            mbar_init(&S.d_full[s], 1);
            mbar_init(&S.d_empty[s], kWorkers);
            mbar_init(&S.comb_full[s], kWorkers / 2);
            mbar_init(&S.comb_empty[s], kWorkers / 2);
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
        Seq q{};
        q.start(P);
        for (; q.item >= 0; q.next(P)) {
            const TProblem &pr = P.p[q.prob];
            const int slot = prod_issued % kRS;
            const uint32_t g = prod_issued;
            bool ok = true;
            if (lane == 0) ok = wait_or_abort(&S.raw_empty[slot], ((g / kRS) & 1) ^ 1, S, P.err);
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
        // (every copy issued here is waited for by the workers, or by the
        // bounded waits of the abort path below, before the CTA exits)
    } else if (warp == kWarpMMA) {
        if (lane == 0) {
            uint32_t g = 0;
            Seq q{};
            q.start(P);
            for (; q.item >= 0; q.next(P), ++g) {
                const int buf = g & 1;
                if (!wait_or_abort(&S.ab_full[buf], (g >> 1) & 1, S, P.err)) break;
                if (!wait_or_abort(&S.b_full[buf], (g >> 1) & 1, S, P.err)) break;
                if (!wait_or_abort(&S.d_empty[buf], ((g >> 1) & 1) ^ 1, S, P.err)) break;
                tc_fence_after();
                const uint64_t bdesc = sw128_kmajor_desc(smem_addr(S.b[buf]));
                #pragma unroll
                for (int i = 0; i < 8; ++i)
                    #pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        // block i = k [32i, 32i+32): swizzle atom i/2, byte offset 64*(i%2) + 32*j in its rows
                        const uint32_t off = (i >> 1) * 2048 + (i & 1) * 64 + j * 32;
                        tc_mma_ts(tmem + kDCol + 128 * buf + 16 * i, tmem + kACol + 128 * buf + 16 * i + 8 * j,
                                  bdesc + (off >> 4), kIdesc, j);
                    }
                tc_commit(&S.d_full[buf]);
                tc_commit(&S.b_empty[buf]);
            }
            tc_commit(&S.mma_done);
            if (!wait_or_abort(&S.mma_done, 0, S, P.err)) mbar_wait(&S.mma_done, 0, P.err);
        }
    } else if (warp == kWarpX) {
        // ---------------------------------------------------------------- X rows -> B operand
        uint32_t g = 0;
        Seq q{};
        q.start(P);
        for (; q.item >= 0; q.next(P), ++g) {
            const TProblem &pr = P.p[q.prob];
            const int slot = g % kRS, buf = g & 1;
            bool ok = true;
            if (lane == 0) {
                ok = wait_or_abort(&S.raw_full[slot], (g / kRS) & 1, S, P.err);
                // B[buf] was last read by the MMAs of stage g-2
                if (ok) ok = wait_or_abort(&S.b_empty[buf], ((g >> 1) & 1) ^ 1, S, P.err);
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            // 128-byte swizzle; k permuted within 4-groups as in the A operand
            for (int c = lane; c < pr.M * 32; c += 32) {
                const int m = c >> 5, kc = c & 31;
                const uint4 v = *reinterpret_cast<const uint4 *>(S.raw[slot] + kRawW + m * kXRow + kc * 16);
                uint4 o;
                o.x = prmt(v.x, v.y, 0x5410u);   // (x0, x2)
                o.y = prmt(v.x, v.y, 0x7632u);   // (x1, x3)
                o.z = prmt(v.z, v.w, 0x5410u);   // (x4, x6)
                o.w = prmt(v.z, v.w, 0x7632u);   // (x5, x7)
                *reinterpret_cast<uint4 *>(S.b[buf] + (kc >> 3) * 2048 + (m >> 3) * 1024 + (m & 7) * 128 +
                                           (((kc & 7) ^ (m & 7)) * 16)) = o;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&S.b_full[buf]);
                mbar_arrive(&S.raw_empty[slot]);
            }
        }
    } else {
        // ---------------------------------------------------------------- workers
        const int quad = warp & 3;            // tensor-memory lanes 32*quad ..
        const int half = (warp - kWarp0) >> 2;   // blocks 4*half .. 4*half+3 of each stage
        const uint32_t lane_base = uint32_t(32 * quad) << 16;
        float acc[MP];
        #pragma unroll
        for (int m = 0; m < MP; ++m) acc[m] = 0.f;
        // stages g-1 and g-2 still owe their scaling: a two-entry ring
        struct Pending {
            float d[4];
            int last, prob, row0;
        };
        Pending pend[2];
        uint32_t items_done = 0;
        bool ok = true;

        // read back stage gp's per-block sums, scale by d, and finish the item if it was its last stage
        auto scale = [&](uint32_t gp) -> bool {
            const int buf = gp & 1;
            const Pending &pd = pend[gp & 1];
            if (!wait_or_abort(&S.d_full[buf], (gp >> 1) & 1, S, P.err)) return false;
            tc_fence_after();
            if constexpr (MP <= 4) {   // four loads in flight, one wait
                float v[4][MP];
                #pragma unroll
                for (int jb = 0; jb < 4; ++jb)
                    tc_ld_cols<MP>(tmem + lane_base + kDCol + 128 * buf + 16 * (4 * half + jb), v[jb]);
                tc_wait_ld();
                #pragma unroll
                for (int jb = 0; jb < 4; ++jb)
                    #pragma unroll
                    for (int m = 0; m < MP; ++m) acc[m] = fmaf(pd.d[jb], v[jb][m], acc[m]);
            } else {
                #pragma unroll
                for (int jb = 0; jb < 4; ++jb) {
                    float v[MP];
                    tc_ld_cols<MP>(tmem + lane_base + kDCol + 128 * buf + 16 * (4 * half + jb), v);
                    tc_wait_ld();
                    #pragma unroll
                    for (int m = 0; m < MP; ++m) acc[m] = fmaf(pd.d[jb], v[m], acc[m]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.d_empty[buf]);
            if (pd.last) {
                const TProblem &pr = P.p[pd.prob];
                const int cb = items_done & 1;
                const uint32_t par = (items_done >> 1) & 1;
                if (half == 1) {
                    if (!wait_or_abort(&S.comb_empty[cb], par ^ 1, S, P.err)) return false;
                    #pragma unroll
                    for (int m = 0; m < MP; ++m) S.comb[cb][quad][m][lane] = acc[m];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.comb_full[cb]);
                } else {
                    if (!wait_or_abort(&S.comb_full[cb], par, S, P.err)) return false;
                    #pragma unroll
                    for (int m = 0; m < MP; ++m) acc[m] += S.comb[cb][quad][m][lane];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.comb_empty[cb]);
                    const int n = pd.row0 + 32 * quad + lane;
                    if (n < pr.N) {
                        #pragma unroll
                        for (int m = 0; m < MP; ++m)
                            if (m < pr.M) pr.Y[static_cast<int64_t>(m) * pr.N + n] = acc[m];
                    }
                }
                #pragma unroll
                for (int m = 0; m < MP; ++m) acc[m] = 0.f;
                ++items_done;
            }
            return true;
        };

        uint32_t g = 0;
        Seq q{};
        q.start(P);
        for (; q.item >= 0; q.next(P), ++g) {
            const TProblem &pr = P.p[q.prob];
            const int slot = g % kRS, buf = g & 1;
            if (!(ok = wait_or_abort(&S.raw_full[slot], (g / kRS) & 1, S, P.err))) break;
            // this thread's half row: bytes [64*half, 64*half + 80) of the 144-byte stage row
            uint32_t w[20];
            {
                const uint4 *src = reinterpret_cast<const uint4 *>(S.raw[slot] + (32 * quad + lane) * kRawRow + 64 * half);
                #pragma unroll
                for (int i = 0; i < 5; ++i) {
                    const uint4 v = src[i];
                    w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.raw_empty[slot]);

            // Stage g-2: its MMAs were issued a whole iteration ago.  Reading
            // its sums back also frees A[g&1] (the MMAs have finished reading
            // it) and lets the MMAs of stage g reuse D[g&1].
            if (g > 1 && !(ok = scale(g - 2))) break;

            // dequantize blocks 4*half .. 4*half+3 into 64 tensor-memory columns
            uint32_t cols[64];
            Pending &pn = pend[g & 1];
            if (half == 0) dequant_half<0>(w, cols, pn.d);
            else dequant_half<1>(w, cols, pn.d);
            pn.last = (q.stage == q.nstages - 1);
            pn.prob = q.prob;
            pn.row0 = q.row0;
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
            if (lane == 0) mbar_arrive(&S.ab_full[buf]);
        }
        if (ok && g > 1) ok = scale(g - 2);
        if (ok && g > 0) ok = scale(g - 1);
    }

    tc_fence_before();
    __syncthreads();
    // Abort path: copies issued but never consumed may still be in flight;
    // let them land (bounded) before the CTA exits.
    if (*reinterpret_cast<volatile int *>(&S.abort_flag) && warp == kWarpProd && lane == 0) {
        for (uint32_t i = 0; i < kRS && i < prod_issued; ++i) {
            const uint32_t gg = prod_issued - 1 - i;
            mbar_wait(&S.raw_full[gg % kRS], (gg / kRS) & 1, P.err);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMMA) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

template <int MP, int CAP>
cudaError_t launch_mp(TParams<CAP> &P, const q4::DeviceInfo &dev, cudaStream_t s) {
    static int configured_device = -1;
    if (configured_device != dev.device) {
        cudaError_t e = cudaFuncSetAttribute(decode_tmem_kernel<MP, CAP>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes));
        if (e != cudaSuccess) return e;
        configured_device = dev.device;
    }
    const int grid = std::max(1, std::min(dev.sm_count, P.total_items));
    decode_tmem_kernel<MP, CAP><<<grid, kThreads, kSmemBytes, s>>>(P);
    return cudaGetLastError();
}

// problems[0..count) sorted by K (largest first), count <= CAP
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
    if (maxM <= 1) return launch_mp<1, CAP>(P, dev, s);
    if (maxM <= 2) return launch_mp<2, CAP>(P, dev, s);
    if (maxM <= 4) return launch_mp<4, CAP>(P, dev, s);
    if (maxM <= 8) return launch_mp<8, CAP>(P, dev, s);
    return launch_mp<16, CAP>(P, dev, s);
}

constexpr int kSmallCap = 8, kLargeCap = 128;

}  // namespace

namespace q4 {

bool decode_tmem_supports(const Problem &p) {
    return p.M >= 1 && p.M <= kMaxM && p.K >= kStageK && p.K % kStageK == 0 && p.N >= 1 && p.N < (1LL << 31) &&
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
