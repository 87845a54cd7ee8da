// q4_0_decode.cu -- the memory-bound decode path (M <= 32): one persistent
// launch streams the Q4_0 weights of one or many problems exactly once from
// HBM, dequantizes them in registers and multiplies with the (tiny) bf16
// activations on the warp-level tensor cores.
//
// The pages' decode loop runs a Q4 matmul for every linear of each of the 26
// decoder layers per token (voxtral-mini-realtime-rs (Shannon-Prime fork)
// README, "Architecture Summary"; decode dominates: "Pipeline Overlap"), with
// batch 2 for CFG and fused QKV / gate-up projections ("TTS (Text-to-Speech)",
// optimizations) and up to 32 concurrent sequences in the Tenstorrent port
// (Voxtral-Mini-4B-Realtime-2602-tt-p300x2 README, serving section).
//
// Design (B200):
//  * every warp is an independent worker with its own ring of shared-memory
//    stages; a stage is 16*RT weight rows x 1024 k (4 groups of 8 blocks =
//    576 contiguous bytes per row), fetched with one 1-D bulk copy
//    (cp.async.bulk, completion on an mbarrier) per row; rows start 16-byte
//    aligned because a row is K/256 * 144 bytes;
//  * work items are (problem, 16*RT rows, all of K); problems are sorted by K
//    (largest first) on the host and items are dealt to the grid's warps in
//    boustrophedon order, so every warp gets a similar byte count;
//  * the 4-bit codes are turned into exact bf16 values (q - 8) with two byte
//    permutes, a mask-or against the bf16 bit pattern of 128 and one packed
//    subtraction per pair of weights; the products with X run on
//    mma.sync.m16n8k16 (bf16 in, fp32 out) with the weight rows as the MMA's
//    M dimension and the (at most 32) rows of X as its N dimension;
//  * each 32-k block is multiplied in its own pair of MMAs and scaled by its
//    fp16 d in fp32 (the scale never rounds a weight); the k order inside a
//    block is permuted identically on both operands so that X is read in its
//    natural row-major layout (8 consecutive bf16 per thread and MMA).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <vector>

#include "q4_0_internal.cuh"

namespace {

using namespace q4dev;

constexpr int kWarps = 8;                 // workers per CTA (1 CTA per SM)
constexpr int kStages = 3;                // ring depth per worker
constexpr int kGroupsPerStage = 4;        // 4 x 256 k per stage
constexpr int kGroupBytes = 144;          // 8 blocks x 18 bytes
constexpr int kRowPitch = kGroupsPerStage * kGroupBytes + 16;   // 592: conflict-free reads
constexpr int kMaxProblems = Q4_0_MAX_GROUP;

struct DecodeProblem {
    const uint8_t *W;
    const uint16_t *X;
    float *Y;
    int M, N, K;
    int groups;        // K / 256
    int item_begin;    // first item index of this problem
};

struct DecodeParams {
    int count;
    int total_items;
    int rows_per_item;
    unsigned *err;
    DecodeProblem p[kMaxProblems];
};

template <int RT>
constexpr int stage_bytes() { return 16 * RT * kRowPitch; }

__device__ __forceinline__ int find_problem(const DecodeParams &P, int item) {
    int lo = 0, hi = P.count - 1;
    while (lo < hi) {   // last problem with item_begin <= item
        const int mid = (lo + hi + 1) >> 1;
        if (P.p[mid].item_begin <= item) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Walks one warp's sequence of (item, k-chunk) stages.
struct Cursor {
    int round;      // deal round
    int item;       // global item index, or -1 when done
    int prob;
    int row0;
    int chunk;
    int nchunks;

    __device__ __forceinline__ void load_item(const DecodeParams &P, int gw, int GW) {
        const int pos = (round & 1) ? (GW - 1 - gw) : gw;
        item = round * GW + pos;
        if (item >= P.total_items) { item = -1; return; }
        prob = find_problem(P, item);
        row0 = (item - P.p[prob].item_begin) * P.rows_per_item;
        chunk = 0;
        nchunks = (P.p[prob].groups + kGroupsPerStage - 1) / kGroupsPerStage;
    }
    __device__ __forceinline__ void start(const DecodeParams &P, int gw, int GW) {
        round = 0;
        load_item(P, gw, GW);
    }
    __device__ __forceinline__ void next(const DecodeParams &P, int gw, int GW) {
        if (++chunk < nchunks) return;
        ++round;
        load_item(P, gw, GW);
    }
};

// Issue the bulk copies of one stage: rows [row0, row0 + 16*RT) x groups
// [chunk*4, chunk*4 + gc) into `dst` (row pitch kRowPitch).
template <int RT>
__device__ __forceinline__ void issue_stage(const DecodeParams &P, const Cursor &c, uint8_t *dst,
                                            uint64_t *full, int lane) {
    const DecodeProblem &pr = P.p[c.prob];
    const int g0 = c.chunk * kGroupsPerStage;
    const int gc = min(kGroupsPerStage, pr.groups - g0);
    const int rows = min(16 * RT, pr.N - c.row0);
    const uint32_t bytes_per_row = static_cast<uint32_t>(gc * kGroupBytes);
    if (lane == 0) mbar_arrive_expect_tx(full, bytes_per_row * static_cast<uint32_t>(rows));
    __syncwarp();
    const int64_t row_bytes = static_cast<int64_t>(pr.groups) * kGroupBytes;
    for (int r = lane; r < rows; r += 32) {
        const uint8_t *src = pr.W + (static_cast<int64_t>(c.row0) + r) * row_bytes +
                             static_cast<int64_t>(g0) * kGroupBytes;
        bulk_g2s(dst + r * kRowPitch, src, bytes_per_row, full);
    }
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                         const float (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

// Exact bf16 pairs (q - 8) from one qs word (bytes b0..b3 of a row's block):
//   lo01 = (q[b0.lo], q[b1.lo]), lo23 = (q[b2.lo], q[b3.lo]),
//   hi01 = (q[b0.hi], q[b1.hi]), hi23 = (q[b2.hi], q[b3.hi]).
// 0x4300 is bf16 128.0 (7 fraction bits, so 128 + q is exact for q < 16);
// subtracting bf16 136.0 leaves q - 8 exactly.
__device__ __forceinline__ void codes_to_bf16(uint32_t v, uint32_t &lo01, uint32_t &lo23, uint32_t &hi01,
                                              uint32_t &hi23) {
    const uint32_t s01 = prmt(v, 0u, 0x4140u);   // bytes [b0, 0, b1, 0]
    const uint32_t s23 = prmt(v, 0u, 0x4342u);   // bytes [b2, 0, b3, 0]
    const __nv_bfloat162 off = __halves2bfloat162(__ushort_as_bfloat16(0x4308), __ushort_as_bfloat16(0x4308));
    uint32_t t;
    t = and_or(s01, 0x000F000Fu, 0x43004300u);
    __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162 *>(&t), off);
    lo01 = *reinterpret_cast<uint32_t *>(&r);
    t = and_or(s23, 0x000F000Fu, 0x43004300u);
    r = __hsub2(*reinterpret_cast<__nv_bfloat162 *>(&t), off);
    lo23 = *reinterpret_cast<uint32_t *>(&r);
    t = and_or(s01 >> 4, 0x000F000Fu, 0x43004300u);
    r = __hsub2(*reinterpret_cast<__nv_bfloat162 *>(&t), off);
    hi01 = *reinterpret_cast<uint32_t *>(&r);
    t = and_or(s23 >> 4, 0x000F000Fu, 0x43004300u);
    r = __hsub2(*reinterpret_cast<__nv_bfloat162 *>(&t), off);
    hi23 = *reinterpret_cast<uint32_t *>(&r);
}

// qs word t (bytes 2+4t .. 5+4t of the block) of the block starting at `blk`.
// Blocks at an even index within a 144-byte group start 4-byte aligned, odd
// ones at 2 mod 4.
__device__ __forceinline__ uint32_t qs_word(const uint8_t *blk, int odd, int t) {
    if (odd) {
        return *reinterpret_cast<const uint32_t *>(blk + 2 + 4 * t);
    } else {
        const uint32_t lo = *reinterpret_cast<const uint32_t *>(blk + 4 * t);
        const uint32_t hi = *reinterpret_cast<const uint32_t *>(blk + 4 * t + 4);
        return prmt(lo, hi, 0x5432u);
    }
}

template <int NT, int RT>
__global__ void __launch_bounds__(kWarps * 32, 1) decode_kernel(const __grid_constant__ DecodeParams P) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int GW = gridDim.x * kWarps;
    const int gw = blockIdx.x * kWarps + warp;

    constexpr int SB = stage_bytes<RT>();
    uint8_t *ring = smem + static_cast<size_t>(warp) * kStages * SB;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + static_cast<size_t>(kWarps) * kStages * SB) +
                     warp * kStages;
    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    Cursor issue, cons;
    issue.start(P, gw, GW);
    cons = issue;
    uint32_t issued = 0;
    for (int s = 0; s < kStages && issue.item >= 0; ++s) {
        issue_stage<RT>(P, issue, ring + s * SB, &full[s], lane);
        issue.next(P, gw, GW);
        ++issued;
    }

    float acc[RT][NT][4];
    uint32_t consumed = 0;
    while (cons.item >= 0) {
        const int s = consumed % kStages;
        const uint32_t parity = (consumed / kStages) & 1;
        if (!mbar_wait(&full[s], parity, P.err)) {
            // Gave up (error word set).  Wait, again with a bound, for the
            // copies this warp still has in flight, then leave.
            for (uint32_t j = consumed + 1; j < issued; ++j)
                if (!mbar_wait(&full[j % kStages], (j / kStages) & 1, P.err)) break;
            return;
        }

        const DecodeProblem &pr = P.p[cons.prob];
        if (cons.chunk == 0) {
            #pragma unroll
            for (int r = 0; r < RT; ++r)
                #pragma unroll
                for (int j = 0; j < NT; ++j)
                    #pragma unroll
                    for (int e = 0; e < 4; ++e) acc[r][j][e] = 0.f;
        }
        const int g0 = cons.chunk * kGroupsPerStage;
        const int gc = min(kGroupsPerStage, pr.groups - g0);
        // X rows used by this thread as MMA column g of n-tile j (rows past M
        // repeat the last row; their outputs are never stored).
        const uint16_t *xrow[NT];
        #pragma unroll
        for (int j = 0; j < NT; ++j)
            xrow[j] = pr.X + static_cast<int64_t>(min(8 * j + g, pr.M - 1)) * pr.K;
        uint8_t *stage = ring + s * SB;

        for (int grp = 0; grp < gc; ++grp) {
            const int kb0 = (g0 + grp) * 8;   // first block index (along K) of this group
            #pragma unroll
            for (int i = 0; i < 8; ++i) {
                // activations of block kb0+i: 2 x 8 bytes per n-tile
                uint2 xb[NT][2];
                #pragma unroll
                for (int j = 0; j < NT; ++j) {
                    const uint16_t *xp = xrow[j] + (kb0 + i) * 32 + 4 * t;
                    xb[j][0] = __ldg(reinterpret_cast<const uint2 *>(xp));
                    xb[j][1] = __ldg(reinterpret_cast<const uint2 *>(xp + 16));
                }
                #pragma unroll
                for (int r = 0; r < RT; ++r) {
                    const uint8_t *bg = stage + (16 * r + g) * kRowPitch + grp * kGroupBytes + 18 * i;
                    const uint8_t *bg8 = bg + 8 * kRowPitch;
                    const float dg = __half2float(*reinterpret_cast<const __half *>(bg));
                    const float dg8 = __half2float(*reinterpret_cast<const __half *>(bg8));
                    const uint32_t qg = qs_word(bg, i & 1, t);
                    const uint32_t qg8 = qs_word(bg8, i & 1, t);
                    uint32_t a0[4], a1[4];
                    // MMA 0: k-cols (2t,2t+1) <- elements (4t,4t+1); (2t+8,2t+9) <- (4t+2,4t+3)
                    // MMA 1: the same with elements + 16 (high nibbles)
                    codes_to_bf16(qg, a0[0], a0[2], a1[0], a1[2]);
                    codes_to_bf16(qg8, a0[1], a0[3], a1[1], a1[3]);
                    #pragma unroll
                    for (int j = 0; j < NT; ++j) {
                        const float z[4] = {0.f, 0.f, 0.f, 0.f};
                        float c[4];
                        mma_bf16(c, a0, xb[j][0].x, xb[j][0].y, z);
                        mma_bf16(c, a1, xb[j][1].x, xb[j][1].y, c);
                        acc[r][j][0] = fmaf(dg, c[0], acc[r][j][0]);
                        acc[r][j][1] = fmaf(dg, c[1], acc[r][j][1]);
                        acc[r][j][2] = fmaf(dg8, c[2], acc[r][j][2]);
                        acc[r][j][3] = fmaf(dg8, c[3], acc[r][j][3]);
                    }
                }
            }
        }

        if (cons.chunk == cons.nchunks - 1) {
            // Y[m, n]: thread holds (row g / g+8, columns 8j+2t, 8j+2t+1)
            #pragma unroll
            for (int r = 0; r < RT; ++r) {
                const int n0 = cons.row0 + 16 * r + g;
                #pragma unroll
                for (int j = 0; j < NT; ++j) {
                    const int m0 = 8 * j + 2 * t;
                    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int m = m0 + (e & 1);
                        const int n = n0 + ((e & 2) ? 8 : 0);
                        if (m < pr.M && n < pr.N) pr.Y[static_cast<int64_t>(m) * pr.N + n] = acc[r][j][e];
                    }
                }
            }
        }

        // The stage has been read by every lane: refill it (the proxy fence
        // orders those generic-proxy reads before the async-proxy writes).
        __syncwarp();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (issue.item >= 0) {
            issue_stage<RT>(P, issue, stage, &full[s], lane);
            issue.next(P, gw, GW);
            ++issued;
        }
        cons.next(P, gw, GW);
        ++consumed;
    }
}

template <int NT, int RT>
cudaError_t launch_nt(DecodeParams &P, const q4::DeviceInfo &dev, cudaStream_t s) {
    const size_t smem = static_cast<size_t>(kWarps) * kStages * stage_bytes<RT>() +
                        static_cast<size_t>(kWarps) * kStages * sizeof(uint64_t);
    static q4::DeviceOnce configured;
    cudaError_t e = configured.run(dev.device, [&] {
        return cudaFuncSetAttribute(decode_kernel<NT, RT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem));
    });
    if (e != cudaSuccess) return e;
    P.rows_per_item = 16 * RT;
    // item boundaries per problem
    int items = 0;
    for (int i = 0; i < P.count; ++i) {
        P.p[i].item_begin = items;
        items += (P.p[i].N + 16 * RT - 1) / (16 * RT);
    }
    P.total_items = items;
    const int need = (items + kWarps - 1) / kWarps;
    const int grid = std::max(1, std::min(dev.sm_count, need));
    decode_kernel<NT, RT><<<grid, kWarps * 32, smem, s>>>(P);
    return cudaGetLastError();
}

}  // namespace

namespace q4 {

bool decode_supports(const Problem &p) {
    return p.M >= 1 && p.M <= 32 && p.K >= 256 && p.K % 256 == 0 && p.N >= 1 && p.N < (1LL << 31) &&
           p.K < (1LL << 31) && (reinterpret_cast<uintptr_t>(p.W) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(p.X) & 15) == 0;
}

cudaError_t launch_decode(const Problem *probs, int count, const DeviceInfo &dev, cudaStream_t s) {
    if (count <= 0) return cudaSuccess;
    // sort by K (largest first) so the deal hands out the long rows first
    std::vector<int> order(count);
    for (int i = 0; i < count; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return probs[a].K > probs[b].K; });
    static thread_local DecodeParams P;
    P.count = count;
    P.err = dev.err;
    int64_t maxM = 1;
    for (int i = 0; i < count; ++i) {
        const Problem &q = probs[order[i]];
        P.p[i].W = q.W;
        P.p[i].X = q.X;
        P.p[i].Y = q.Y;
        P.p[i].M = static_cast<int>(q.M);
        P.p[i].N = static_cast<int>(q.N);
        P.p[i].K = static_cast<int>(q.K);
        P.p[i].groups = static_cast<int>(q.K / 256);
        maxM = std::max(maxM, q.M);
    }
    if (maxM <= 8) return launch_nt<1, 1>(P, dev, s);
    if (maxM <= 16) return launch_nt<2, 1>(P, dev, s);
    return launch_nt<4, 1>(P, dev, s);
}

}  // namespace q4
