// q4_0_decode_mma.cu -- the memory-bound decode path (M <= 32): one
// persistent launch streams the Q4_0 weights of one or many problems once
// from HBM, dequantizes them in registers and multiplies them with the few
// activation rows on the warp-level tensor cores (mma.sync).
//
// The pages' token loop runs a Q4 matmul for every decoder linear of each of
// the 26 layers (voxtral-mini-realtime-rs (Shannon-Prime fork) README,
// "Architecture Summary"; decode is most of the time: "Pipeline Overlap"),
// with batch-2 CFG and fused QKV / gate-up projections ("TTS
// (Text-to-Speech)", optimizations), and up to 32 concurrent sequences in the
// Tenstorrent port (Voxtral-Mini-4B-Realtime-2602-tt-p300x2 README, serving).
//
// Why mma.sync and not tcgen05: a tcgen05.mma with M=128, K=16 takes ~112
// cycles whatever N (measured), so with the weights as its A operand an SM
// turns at most ~18 weights per cycle into products -- about 3 TB/s of Q4_0 on
// B200, half of what HBM delivers.  The warp-level m16n8k16 has no such floor,
// and its n=8 matches the few activation rows.
//
// Per CTA (one per SM): a producer warp and two groups of 8 compute warps;
// compute group G takes the stages g with g mod 2 == G, so that two stages
// are worked on at once.
//  * stage = 256 k of an item (128 weight rows x 144 bytes, one TMA box) plus
//    the same 256 k of every row of X (1-D bulk copies), in a ring of 4-6
//    slots; for M <= 8 a slot holds two stages, so that every wait, arrival
//    and walk step covers 512 k; the TMA box pattern alone streams at
//    ~6.9 TB/s (measured);
//  * compute warp w of a group owns rows 16w .. 16w+15; thread (g, t) reads
//    the 36 contiguous bytes of blocks 2t and 2t+1 of rows g and g+8 (nine
//    conflict-free 4-byte loads per row), turns them into fp16 (q - 8) * d
//    pairs and feeds them as A fragments of 16 mma.sync per stage: with the
//    scale folded into each weight, one MMA may mix blocks, so every byte a
//    thread loads is its own;
//  * for M > 8 the stage's X rows come as four TMA boxes (64 k x 8*NT rows,
//    128-byte swizzle, rows past M zero-filled) instead of one 1-D copy per
//    row: 32 copies per stage would cap the stream near 2.2 TB/s;
//  * the compute warps of the group convert the stage's X rows to fp16
//    straight into the matching mma.sync B fragments (two buffers per
//    group), each warp one eighth of every row, and meet on the buffer's
//    barrier before their MMAs.  The fragments of a code word's two MMAs sit
//    side by side: one 16-byte shared load per pair for the compute threads.
//    (A separate conversion warp per group held the group back at M = 32: it
//    alone issued as many instructions per stage as a compute warp's MMAs and
//    dequantization together.  Warps of 32 rows over half the blocks, which
//    halve the fragment traffic, need the stage's words live across the MMAs:
//    with the producer warp the CTA has 96 registers a thread, and either the
//    words spill or the slot is held until the MMAs end, which starves the
//    ring; both measured slower.)
//  * fused epilogues (decode only): Y = sums + R, or, for a gate/up weight
//    whose items hold 64 gate rows then the same 64 features' up rows,
//    Y[m, f] = silu(gate) * up with the up tiles' sums handed to the gate
//    tiles through shared memory -- the intermediate never reaches HBM;
//  * the accumulators (one chain per n-tile, two for a single n-tile) live
//    across the whole item; at its end the group-1 warp hands its sums
//    through shared memory to the group-0 warp of the same rows, which
//    stores Y[m, n].
// Split mode (M <= 8, up to kMaxItems items): when a launch has few items,
// whole items leave a tail -- one decoder layer at M=1 has 24 items of 32
// stages next to 192 of 12, so the busiest CTA works 32 stages against a
// mean of 21 -- and with fewer items than SMs most SMs idle (a 3072 x 3072
// GEMV has 24 items of 12 stages).  The CTAs then run in clusters of CL: two
// when there is at least one item per SM, else 4, 6 or 8, whichever leaves
// the least work on the busiest CTA.  An item longer than the mean load of
// a CTA is split: the CL CTAs of a cluster take its CL pieces, all first
// thing, and the sums of ranks 1..CL-1 reach rank 0 through distributed
// shared memory before it stores Y.  The other items stay whole, each on
// one CTA.  The host deals the split items to the clusters and then the
// whole items to the CTAs, longest first onto the least loaded.
// Launches use programmatic stream serialization: the next grid on the
// stream may start as this grid's CTAs leave, and every CTA waits for the
// previous grid before its first global access.
// Numerics: each weight is rounded once to fp16 (relative error <= 2^-11,
// inside the 1e-3 tolerance of the method); X is exact in fp16 within its
// normal range; products are exact and accumulation is fp32.  Operands beyond
// the fp16 range (|x| > 65504, |d| > 8188) overflow to +-inf.
#include <cuda_fp16.h>

#include <algorithm>
#include <vector>

#include "q4_0_convert.cuh"
#include "q4_0_internal.cuh"
#include "q4_0_sched.cuh"
#include "q4_0_split_plan.h"
#include "q4_0_tcgen05.cuh"
#include "q4_0_tmap.cuh"

namespace {

using namespace q4dev;

constexpr int kRawW = kItemRows * kStageRowBytes;   // 18432
constexpr int kXRow = kStageK * 2;                  // 512 bytes of one bf16 X row per stage
constexpr int kXPitch = kXRow + 16;                 // skews consecutive X rows by four banks
constexpr int kXBufs = 4;                           // buffer g mod 4 belongs to group g mod 2
constexpr int kWarpProd = 0, kWarp0 = 1, kGroupWarps = 8;
constexpr int kThreads = 32 * (kWarp0 + 2 * kGroupWarps);  // 544
using q4split::kMaxItems;
using q4split::kMaxSched;
using q4split::kMaxSplitCtas;
using q4split::kSplitFlag;

// NT = n8 tiles of X rows (M <= 8*NT)
// X by TMA boxes (M > 8): four boxes of 64 k x 8*NT rows, 128 bytes a row
template <int NT> constexpr bool xmap() { return NT >= 2; }
template <int NT> constexpr int xbox_bytes() { return 8 * NT * 128; }
template <int NT> constexpr int raw_bytes() {   // one 256-k stage
    return kRawW + (xmap<NT>() ? 4 * xbox_bytes<NT>() : 8 * NT * kXPitch);
}
// 256-k stages per ring slot: two for M <= 8, so that every wait, arrival and
// walk step of every warp covers 512 k (halving that overhead per byte)
template <int NT> constexpr int subs() { return NT == 1 ? 2 : 1; }
// ring slots; clusters of CL >= 4 (launches of few items, where a CTA works
// a few stages) give part of the ring to the partner sums
template <int NT, int CL> constexpr int ring() { return CL >= 6 ? 2 : CL == 4 ? 3 : NT == 2 ? 6 : 4; }

// Partner sums in split mode: rank r > 0 of a cluster of CL writes its
// sums remotely into slot r - 1 of rank 0's copy (two buffers, by item
// parity).
template <int NT, int CL>
struct XComb {
    float v[2][CL - 1][8][NT][4][32];
    uint64_t full[2], empty[2];
};
template <int NT>
struct XComb<NT, 1> {};

template <int NT, int CL>
struct Smem {
    uint8_t raw[ring<NT, CL>()][subs<NT>()][raw_bytes<NT>()];   // per stage: W rows (pitch 144), X rows (pitch 528)
    uint4 xf[kXBufs][subs<NT>()][8][NT][32];                // B fragments of MMAs 2v, 2v+1: [stage][v][n tile][lane]
    float comb[8][NT][4][32];                   // group-1 sums handed to group 0 at an item's end
    uint64_t raw_full[ring<NT, CL>()], raw_empty[ring<NT, CL>()];
    uint64_t xf_full[kXBufs];
    uint64_t comb_full, comb_empty;
    float epi[4][NT][4][32];                    // SwiGLU: up-row sums handed to the gate rows
    uint64_t epi_full, epi_empty;
    XComb<NT, CL> x;
    int abort_flag;
};

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint2 b) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y));
}

// One row's blocks 2t and 2t+1 of a stage: the 36 bytes at 36t of the
// 144-byte row, as nine 4-byte words r[0..8].  Block 2t starts 4-byte
// aligned (scale = low half of r[0], codes straddle words), block 2t+1 at
// 2 mod 4 (scale = high half of r[4], codes in r[5..8]).
__device__ __forceinline__ void load_blocks(const uint8_t *row, int t, uint32_t (&r)[9]) {
    const uint32_t *p = reinterpret_cast<const uint32_t *>(row + 36 * t);
    #pragma unroll
    for (int i = 0; i < 9; ++i) r[i] = p[i];
}

// (d, d) and code word w of block b (0: block 2t, 1: block 2t+1).
template <int B>
__device__ __forceinline__ void block_word(const uint32_t (&r)[9], int w, uint32_t &d2, uint32_t &qw) {
    if constexpr (B == 0) {
        d2 = prmt(r[0], r[0], 0x1010u);
        qw = prmt(r[w], r[w + 1], 0x5432u);
    } else {
        d2 = prmt(r[4], r[4], 0x3232u);
        qw = r[5 + w];
    }
}

// MMAs u = 8B + 2w (low nibbles) and u + 1 (high nibbles) of the stage.
// Accumulator chains per n-tile: with one n-tile, the low- and high-nibble
// MMAs of a code word go to two chains so that they do not wait on each
// other; with 2 or 4 n-tiles one chain each, the low-nibble MMAs of all
// n-tiles issued before the high-nibble ones (a chain's MMAs NT apart), which
// frees NT * 4 registers (M = 32: 2.09 -> 2.21 TB/s).
template <int NT> constexpr int chains() { return NT == 1 ? 2 : 1; }

template <int NT, int B, int W>
__device__ __forceinline__ void word_mma(const uint32_t (&rg)[9], const uint32_t (&rg8)[9],
                                         const uint4 (&xf)[8][NT][32], int lane,
                                         float (&acc)[chains<NT>()][NT][4]) {
    uint32_t dg, dg8, qg, qg8;
    block_word<B>(rg, W, dg, qg);
    block_word<B>(rg8, W, dg8, qg8);
    uint32_t cg[4], cg8[4];
    q4_word_to_fp16(qg, dg, cg);
    q4_word_to_fp16(qg8, dg8, cg8);
    constexpr int u = 8 * B + 2 * W;
    constexpr int C = chains<NT>();
    // one 16-byte load per n-tile: the fragments of MMAs u and u + 1
    uint4 b[NT];
    #pragma unroll
    for (int j = 0; j < NT; ++j) b[j] = xf[u >> 1][j][lane];
    // a0/a1: k cols (2t, 2t+1) of rows g / g+8; a2/a3: k cols (2t+8, 2t+9)
    if constexpr (C == 2) {
        #pragma unroll
        for (int j = 0; j < NT; ++j) {
            mma_f16(acc[0][j], cg[0], cg8[0], cg[1], cg8[1], make_uint2(b[j].x, b[j].y));
            mma_f16(acc[1][j], cg[2], cg8[2], cg[3], cg8[3], make_uint2(b[j].z, b[j].w));
        }
    } else {
        #pragma unroll
        for (int j = 0; j < NT; ++j) mma_f16(acc[0][j], cg[0], cg8[0], cg[1], cg8[1], make_uint2(b[j].x, b[j].y));
        #pragma unroll
        for (int j = 0; j < NT; ++j) mma_f16(acc[0][j], cg[2], cg8[2], cg[3], cg8[3], make_uint2(b[j].z, b[j].w));
    }
}

constexpr int kXMapCap = 64;   // problems per launch when X maps are passed (M > 8)

template <int CAP>
struct DecodeParams {
    GroupParams<CAP> g;
    CUtensorMap xmap[CAP <= kXMapCap ? CAP : 1];   // M > 8: X as bf16 [M, K], box 64 x 8*NT, 128-byte swizzle
    // split mode: CTA b runs sched[sched_begin[b] .. sched_begin[b+1]), each
    // entry an item index, with kSplitFlag set for a piece of a split item
    uint16_t sched_begin[kMaxSplitCtas + 1];
    uint16_t sched[kMaxSched];
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t remote_addr(const void *local, uint32_t rank) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_addr(local)), "r"(rank));
    return ra;
}

__device__ __forceinline__ void st_remote(float *local, uint32_t rank, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote_addr(local, rank)), "f"(v) : "memory");
}

__device__ __forceinline__ void mbar_arrive_remote(uint64_t *local, uint32_t rank) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_addr(local, rank))
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// wait_or_abort for a barrier that another CTA of the cluster arrives on.
__device__ __forceinline__ bool wait_cluster_or_abort(uint64_t *bar, uint32_t parity, int *abort_flag,
                                                      unsigned *err) {
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait_cluster(bar, parity)) {
        if (*reinterpret_cast<volatile int *>(abort_flag)) return false;
        if (global_ns() - t0 > kWaitLimitNs) {
            atomicOr(err, (unsigned)Q4_DEVERR_WAIT_TIMEOUT);
            *reinterpret_cast<volatile int *>(abort_flag) = 1;
            return false;
        }
    }
    return true;
}

// One CTA's walk over its (item, stage) sequence.  Plain mode (CL = 1): the
// items dealt to the CTAs in boustrophedon order.  Split mode: the CTA's list
// from the host; of a split n-stage item rank r of the cluster of CL takes
// stages ceil(n r / CL) .. ceil(n (r + 1) / CL) - 1 (at least one: the host
// splits only items of n >= CL stages).
template <int CL, int SUBS>
struct Walk {
    int round, idx, item, prob, row0, stage, end, cnt;   // this step covers stages [stage, stage + cnt)
    bool split;
    template <int CAP>
    __device__ __forceinline__ void load(const DecodeParams<CAP> &D, uint32_t rank) {
        const GroupParams<CAP> &P = D.g;
        if constexpr (CL == 1) {
            const int G = gridDim.x;
            const int pos = (round & 1) ? (G - 1 - static_cast<int>(blockIdx.x)) : static_cast<int>(blockIdx.x);
            item = round * G + pos;
            if (item >= P.total_items) { item = -1; return; }
            prob = find_problem(P, item);
            stage = 0;
            end = P.p[prob].stages;
            split = false;
        } else {
            if (idx >= D.sched_begin[blockIdx.x + 1]) { item = -1; return; }
            const uint16_t e = D.sched[idx];
            item = e & (kSplitFlag - 1);
            split = (e & kSplitFlag) != 0;
            prob = find_problem(P, item);
            const int n = P.p[prob].stages;
            stage = split ? q4split::piece_begin(n, static_cast<int>(rank), CL) : 0;
            end = split ? q4split::piece_begin(n, static_cast<int>(rank) + 1, CL) : n;
        }
        row0 = (item - P.p[prob].item_begin) * kItemRows;
        cnt = SUBS == 1 || end - stage >= SUBS ? SUBS : end - stage;   // every item has >= 1 stage here
    }
    template <int CAP>
    __device__ __forceinline__ void start(const DecodeParams<CAP> &D, uint32_t rank) {
        round = 0;
        idx = 0;
        if constexpr (CL > 1) idx = D.sched_begin[blockIdx.x];
        load(D, rank);
    }
    template <int CAP>
    __device__ __forceinline__ void next(const DecodeParams<CAP> &D, uint32_t rank) {
        stage += cnt;
        if (stage < end) {
            cnt = SUBS == 1 || end - stage >= SUBS ? SUBS : end - stage;
            return;
        }
        ++round;
        ++idx;
        load(D, rank);
    }
};

template <int NT, int CAP, int CL>
__global__ void __launch_bounds__(kThreads, 1) decode_mma_kernel(const __grid_constant__ DecodeParams<CAP> D) {
    constexpr int RS = ring<NT, CL>();
    constexpr int SUB = subs<NT>();
    const GroupParams<CAP> &P = D.g;
    extern __shared__ uint8_t smem_raw[];
    using SM = Smem<NT, CL>;
    SM &S = *reinterpret_cast<SM *>(align_smem<1024>(smem_raw));   // swizzled X boxes want 1024
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < RS; ++s) {
            mbar_init(&S.raw_full[s], 1);
            mbar_init(&S.raw_empty[s], kGroupWarps);
        }
        for (int s = 0; s < kXBufs; ++s) mbar_init(&S.xf_full[s], kGroupWarps);
        mbar_init(&S.comb_full, kGroupWarps);
        mbar_init(&S.comb_empty, kGroupWarps);
        mbar_init(&S.epi_full, kGroupWarps / 2);
        mbar_init(&S.epi_empty, kGroupWarps / 2);
        if constexpr (CL > 1) {
            for (int s = 0; s < 2; ++s) {
                mbar_init(&S.x.full[s], 32 * kGroupWarps * (CL - 1));   // every group-0 thread of ranks 1..CL-1
                mbar_init(&S.x.empty[s], 32 * kGroupWarps);             // every group-0 thread of rank 0
            }
        }
        S.abort_flag = 0;
        fence_mbar_init();
    }
    uint32_t rank = 0;
    if constexpr (CL > 1) {
        rank = cluster_rank();
        cluster_sync_all();   // every CTA's barriers exist before any other CTA arrives on them
    } else {
        __syncthreads();
    }
    // Programmatic dependent launch: the next kernel on the stream may start
    // its CTAs as this grid's CTAs leave the SMs, and this grid reads nothing
    // into the SM before the previous kernel on the stream has completed
    // (both are no-ops for launches without the attribute).  Before that
    // wait the producer only asks L2 for the weight tiles of the CTA's first
    // ring of stages: L2 is where every SM's writes land, so a tile that the
    // previous kernel still writes is current by the time this grid reads it.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == kWarpProd && lane == 0) {
        Walk<CL, SUB> q{};
        q.start(D, rank);
        int prob = -1;
        for (int s = 0; s < RS && q.item >= 0; ++s, q.next(D, rank)) {
            if (q.prob != prob) prefetch_tensormap(&P.wmap[q.prob]);
            prob = q.prob;
            for (int i = 0; i < q.cnt; ++i)
                tma_prefetch_l2_2d(&P.wmap[q.prob], (q.stage + i) * kStageRowBytes, q.row0);
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    uint32_t prod_issued = 0;

    if (warp == kWarpProd) {
        // ---------------------------------------------------------------- loads
        Walk<CL, SUB> q{};
        q.start(D, rank);
        for (; q.item >= 0; q.next(D, rank)) {
            const GroupProblem &pr = P.p[q.prob];
            const uint32_t g = prod_issued;
            const int slot = g % RS;
            bool ok = true;
            if (lane == 0) ok = wait_or_abort(&S.raw_empty[slot], ((g / RS) & 1) ^ 1, &S.abort_flag, P.err);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            // weights: one TMA box per stage (rows past N are zero-filled and still counted)
            if constexpr (xmap<NT>()) {
                if (lane == 0) {
                    // full boxes are counted, zero-filled rows included
                    mbar_arrive_expect_tx(&S.raw_full[slot], q.cnt * (kRawW + 4 * xbox_bytes<NT>()));
                    for (int i = 0; i < q.cnt; ++i) {
                        tma_load_2d(S.raw[slot][i], &P.wmap[q.prob], (q.stage + i) * kStageRowBytes, q.row0,
                                    &S.raw_full[slot]);
                        for (int b = 0; b < 4; ++b)
                            tma_load_2d(S.raw[slot][i] + kRawW + b * xbox_bytes<NT>(), &D.xmap[q.prob],
                                        (q.stage + i) * kStageK + 64 * b, 0, &S.raw_full[slot]);
                    }
                }
            } else {
                if (lane == 0) {
                    mbar_arrive_expect_tx(&S.raw_full[slot], q.cnt * (kRawW + pr.M * kXRow));
                    for (int i = 0; i < q.cnt; ++i)
                        tma_load_2d(S.raw[slot][i], &P.wmap[q.prob], (q.stage + i) * kStageRowBytes, q.row0,
                                    &S.raw_full[slot]);
                }
                __syncwarp();
                for (int i = 0; i < q.cnt; ++i)
                    for (int m = lane; m < pr.M; m += 32)
                        bulk_g2s(S.raw[slot][i] + kRawW + m * kXPitch,
                                 pr.X + static_cast<int64_t>(m) * pr.K + static_cast<int64_t>(q.stage + i) * kStageK,
                                 kXRow, &S.raw_full[slot]);
            }
            ++prod_issued;
        }
    } else {
        // ---------------------------------------------------------------- compute
        const int cw = warp - kWarp0;
        const int G = cw >> 3, tile = cw & 7;   // stage parity, rows 16*tile .. 16*tile+15
        const int gq = lane >> 2, t = lane & 3;
        // X conversion: the B fragment of lane 4gx + tx holds X row 8j + gx at
        // blocks 2tx and 2tx+1 of the stage.  The 16-byte chunk (xw, h, wp) of
        // a row -- k = 32(2tx + xw) + 16h + 8wp .. +7 -- feeds fragments
        // 8xw + 4wp + h (low half) and 8xw + 4wp + 2 + h (high half), i.e. half h
        // of fragment pairs 4xw + 2wp and 4xw + 2wp + 1.  Warp `tile` takes
        // (xw, wp) = (tile >> 2, (tile >> 1) & 1) and the fragment lanes of half
        // s = tile & 1; lane L takes h = L & 1 and, with i = (L >> 1) & 3,
        // c = (L >> 3) & 1 and k = 2s + (L >> 4), gx = (i & 1) + 4 (i >> 1) + 2c
        // and tx = (k + (i >> 1) + 2c) & 3.  Then the eight lanes of each
        // quarter-warp load from eight distinct bank groups (in the swizzled
        // boxes and at the 528-byte pitch alike), and the two lanes of each
        // fragment pair fill it whole, eight pairs with distinct bank groups per
        // half-warp: both the loads and the stores are free of bank conflicts.
        const int xw = tile >> 2, xp = (tile >> 1) & 1, xh = lane & 1;
        const int xi = (lane >> 1) & 3, xc = (lane >> 3) & 1, xq = 2 * (tile & 1) + (lane >> 4);
        const int gx = (xi & 1) + 4 * (xi >> 1) + 2 * xc, tx = (xq + (xi >> 1) + 2 * xc) & 3;
        const int xl = 4 * gx + tx, xu = 8 * xw + 4 * xp + xh;
        const int xk = 32 * (2 * tx + xw) + 16 * xh + 8 * xp;
        uint32_t xbad = 0;
        constexpr int C = chains<NT>();
        float acc[C][NT][4];
        #pragma unroll
        for (int c = 0; c < C; ++c)
            #pragma unroll
            for (int j = 0; j < NT; ++j) acc[c][j][0] = acc[c][j][1] = acc[c][j][2] = acc[c][j][3] = 0.f;
        uint32_t g = 0, items_done = 0, split_done = 0, swiglu_done = 0;
        Walk<CL, SUB> q{};
        q.start(D, rank);
        for (; q.item >= 0; q.next(D, rank), ++g) {
            if ((g & 1) == static_cast<uint32_t>(G)) {
                const int slot = g % RS, xb = g % kXBufs;
                if (!wait_or_abort(&S.raw_full[slot], (g / RS) & 1, &S.abort_flag, P.err)) break;
                // this warp's share of the slot's X -> B fragments.  Buffer xb was
                // last read by the group's slot g - 4; every warp of the group
                // finished that before it arrived on the buffer barrier of slot
                // g - 2, which this warp has passed.
                {
                    const GroupProblem &pr = P.p[q.prob];
                    // every problem's X is range-checked once, by the CTA (or
                    // cluster) that works its first item
                    const bool check = q.row0 == 0;
                    #pragma unroll
                    for (int i = 0; i < SUB; ++i) {
                        if (i >= q.cnt) break;
                        const uint8_t *xr = S.raw[slot][i] + kRawW;
                        #pragma unroll
                        for (int j = 0; j < NT; ++j) {
                            const int m = 8 * j + gx;
                            uint4 o = make_uint4(0u, 0u, 0u, 0u);
                            // TMA boxes (M > 8) zero-fill the rows past M, so every row
                            // converts unconditionally (straight-line loads); 1-D copies
                            // (M <= 8) leave those rows stale
                            if (xmap<NT>() || m < pr.M) {
                                // box tx holds k 64tx..64tx+63; its 16-byte chunk c of row m
                                // sits at chunk c ^ (m & 7) (128-byte swizzle)
                                const uint8_t *src = xmap<NT>()
                                                         ? xr + tx * xbox_bytes<NT>() + m * 128 +
                                                               ((((xk & 63) >> 3) ^ (m & 7)) << 4)
                                                         : xr + m * kXPitch + 2 * xk;
                                const uint4 v = *reinterpret_cast<const uint4 *>(src);
                                if (check) xbad |= x8_fp16_range_bad(v);
                                o = x8_to_fp16_permuted(v);
                            }
                            // fragment u is half u & 1 of pair u >> 1
                            uint2 *f = reinterpret_cast<uint2 *>(&S.xf[xb][i][xu >> 1][j][xl]) + xh;
                            f[0] = make_uint2(o.x, o.y);
                            f[2 * NT * 32] = make_uint2(o.z, o.w);   // fragment xu + 2: the next pair
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.xf_full[xb]);
                uint32_t rg[SUB][9], rg8[SUB][9];
                #pragma unroll
                for (int i = 0; i < SUB; ++i) {
                    if (i >= q.cnt) break;
                    const uint8_t *rowg = S.raw[slot][i] + (16 * tile + gq) * kStageRowBytes;
                    load_blocks(rowg, t, rg[i]);
                    load_blocks(rowg + 8 * kStageRowBytes, t, rg8[i]);
                }
                fence_proxy_async_smem();   // the producer's next copies may land in this slot
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.raw_empty[slot]);
                if (!wait_or_abort(&S.xf_full[xb], (g / kXBufs) & 1, &S.abort_flag, P.err)) break;
                #pragma unroll
                for (int i = 0; i < SUB; ++i) {
                    if (i >= q.cnt) break;
                    word_mma<NT, 0, 0>(rg[i], rg8[i], S.xf[xb][i], lane, acc);
                    word_mma<NT, 0, 1>(rg[i], rg8[i], S.xf[xb][i], lane, acc);
                    word_mma<NT, 0, 2>(rg[i], rg8[i], S.xf[xb][i], lane, acc);
                    word_mma<NT, 0, 3>(rg[i], rg8[i], S.xf[xb][i], lane, acc);
                    word_mma<NT, 1, 0>(rg[i], rg8[i], S.xf[xb][i], lane, acc);
                    word_mma<NT, 1, 1>(rg[i], rg8[i], S.xf[xb][i], lane, acc);
                    word_mma<NT, 1, 2>(rg[i], rg8[i], S.xf[xb][i], lane, acc);
                    word_mma<NT, 1, 3>(rg[i], rg8[i], S.xf[xb][i], lane, acc);
                }
            }
            if (q.stage + q.cnt == q.end) {
                // end of the item: the two groups add their sums
                const GroupProblem &pr = P.p[q.prob];
                const uint32_t par = items_done & 1;
                if (G == 1) {
                    if (!wait_or_abort(&S.comb_empty, par ^ 1, &S.abort_flag, P.err)) break;
                    #pragma unroll
                    for (int j = 0; j < NT; ++j)
                        #pragma unroll
                        for (int e = 0; e < 4; ++e)
                            S.comb[tile][j][e][lane] = C == 2 ? acc[0][j][e] + acc[C - 1][j][e] : acc[0][j][e];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.comb_full);
                } else {
                    if (!wait_or_abort(&S.comb_full, par, &S.abort_flag, P.err)) break;
                    float sum[NT][4];
                    #pragma unroll
                    for (int j = 0; j < NT; ++j)
                        #pragma unroll
                        for (int e = 0; e < 4; ++e)
                            sum[j][e] = (C == 2 ? acc[0][j][e] + acc[C - 1][j][e] : acc[0][j][e]) + S.comb[tile][j][e][lane];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.comb_empty);
                    if constexpr (CL > 1) {
                        if (q.split) {
                            // ranks 1..CL-1 hand their sums to rank 0 of the cluster, which adds
                            // them in rank order
                            const int xb2 = split_done & 1;
                            const uint32_t xpar = (split_done >> 1) & 1;
                            ++split_done;
                            if (rank != 0) {
                                if (!wait_cluster_or_abort(&S.x.empty[xb2], xpar ^ 1, &S.abort_flag, P.err)) break;
                                #pragma unroll
                                for (int j = 0; j < NT; ++j)
                                    #pragma unroll
                                    for (int e = 0; e < 4; ++e)
                                        st_remote(&S.x.v[xb2][rank - 1][tile][j][e][lane], 0, sum[j][e]);
                                mbar_arrive_remote(&S.x.full[xb2], 0);
                            } else {
                                if (!wait_cluster_or_abort(&S.x.full[xb2], xpar, &S.abort_flag, P.err)) break;
                                #pragma unroll
                                for (int r = 0; r < CL - 1; ++r)
                                    #pragma unroll
                                    for (int j = 0; j < NT; ++j)
                                        #pragma unroll
                                        for (int e = 0; e < 4; ++e) sum[j][e] += S.x.v[xb2][r][tile][j][e][lane];
                                #pragma unroll
                                for (int r = 1; r < CL; ++r) mbar_arrive_remote(&S.x.empty[xb2], r);
                            }
                        }
                    }
                    // thread holds rows gq / gq+8 of the tile x columns 8j+2t, 8j+2t+1
                    if (!q.split || rank == 0) {
                        // a non-finite sum from finite inputs means an fp16 weight
                        // overflowed: look at the rows' scales (slow path, rare)
                        bool bad_row[2] = {false, false};
                        #pragma unroll
                        for (int j = 0; j < NT; ++j)
                            #pragma unroll
                            for (int e = 0; e < 4; ++e)
                                if (8 * j + 2 * t + (e & 1) < pr.M && !(fabsf(sum[j][e]) <= 3.402823466e38f))
                                    bad_row[e >> 1] = true;
                        #pragma unroll
                        for (int h = 0; h < 2; ++h)
                            if (bad_row[h]) {
                                const int64_t nn = q.row0 + 16 * tile + gq + 8 * h;
                                scan_scales_fp16_range(pr.W, nn, nn + 1, pr.N, pr.K, P.err);
                            }
                    }
                    if ((!q.split || rank == 0) && pr.epi == kEpiSwiGLU) {
                        // rows 0-63 of the item are gate rows of features row0/2 .. row0/2+63,
                        // rows 64-127 the up rows of the same features: tiles 4-7 hand their
                        // sums to tiles 0-3, which store silu(gate) * up into Y[M, N/2]
                        const uint32_t epar = swiglu_done & 1;
                        ++swiglu_done;
                        if (tile >= 4) {
                            if (!wait_or_abort(&S.epi_empty, epar ^ 1, &S.abort_flag, P.err)) break;
                            #pragma unroll
                            for (int j = 0; j < NT; ++j)
                                #pragma unroll
                                for (int e = 0; e < 4; ++e) S.epi[tile - 4][j][e][lane] = sum[j][e];
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&S.epi_full);
                        } else {
                            if (!wait_or_abort(&S.epi_full, epar, &S.abort_flag, P.err)) break;
                            const int F = pr.N >> 1;
                            #pragma unroll
                            for (int j = 0; j < NT; ++j)
                                #pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float gv = sum[j][e], uv = S.epi[tile][j][e][lane];
                                    const int m = 8 * j + 2 * t + (e & 1);
                                    const int f = (q.row0 >> 1) + 16 * tile + gq + ((e & 2) ? 8 : 0);
                                    if (m < pr.M) pr.Y[static_cast<int64_t>(m) * F + f] = gv / (1.0f + expf(-gv)) * uv;
                                }
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&S.epi_empty);
                        }
                    } else if (!q.split || rank == 0) {
                        #pragma unroll
                        for (int j = 0; j < NT; ++j)
                            #pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int m = 8 * j + 2 * t + (e & 1);
                                const int n = q.row0 + 16 * tile + gq + ((e & 2) ? 8 : 0);
                                if (m < pr.M && n < pr.N) {
                                    const int64_t o = static_cast<int64_t>(m) * pr.N + n;
                                    pr.Y[o] = pr.epi == kEpiResidual ? sum[j][e] + pr.R[o] : sum[j][e];
                                }
                            }
                    }
                }
                #pragma unroll
                for (int c = 0; c < C; ++c)
                    #pragma unroll
                    for (int j = 0; j < NT; ++j) acc[c][j][0] = acc[c][j][1] = acc[c][j][2] = acc[c][j][3] = 0.f;
                ++items_done;
            }
        }
        if (xbad) atomicOr(P.err, (unsigned)Q4_DEVERR_FP16_RANGE);
    }

    __syncthreads();
    // Abort path: copies issued but never consumed may still be in flight;
    // let them land (bounded) before the CTA exits.
    if (*reinterpret_cast<volatile int *>(&S.abort_flag) && warp == kWarpProd && lane == 0) {
        for (uint32_t i = 0; i < RS && i < prod_issued; ++i) {
            const uint32_t gg = prod_issued - 1 - i;
            mbar_wait(&S.raw_full[gg % RS], (gg / RS) & 1, P.err);
        }
    }
    if constexpr (CL > 1) {
        __syncthreads();
        cluster_sync_all();   // no CTA leaves while another CTA of the cluster may still reach its shared memory
    }
}

template <int NT, int CL>
constexpr size_t smem_bytes() { return sizeof(Smem<NT, CL>) + 1024; }
static_assert(smem_bytes<4, 1>() <= 232448, "shared memory budget");
static_assert(smem_bytes<2, 1>() <= 232448, "shared memory budget");
static_assert(smem_bytes<1, 2>() <= 232448, "shared memory budget");
static_assert(smem_bytes<1, 4>() <= 232448, "shared memory budget");
static_assert(smem_bytes<1, 6>() <= 232448, "shared memory budget");
static_assert(smem_bytes<1, 8>() <= 232448, "shared memory budget");

template <int NT, int CAP, int CL>
cudaError_t configure(const q4::DeviceInfo &dev) {
    static q4::DeviceOnce configured;
    return configured.run(dev.device, [] {
        return cudaFuncSetAttribute(decode_mma_kernel<NT, CAP, CL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem_bytes<NT, CL>()));
    });
}

template <int NT, int CAP>
cudaError_t launch_plain(DecodeParams<CAP> &D, const q4::DeviceInfo &dev, cudaStream_t s) {
    cudaError_t e = configure<NT, CAP, 1>(dev);
    if (e != cudaSuccess) return e;
    const int grid = std::max(1, std::min(dev.sm_count, D.g.total_items));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes<NT, 1>();
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_mma_kernel<NT, CAP, 1>, D);
}

template <int CL>
cudaLaunchConfig_t cluster_config(int clusters, cudaStream_t s, cudaLaunchAttribute *attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL * clusters, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes<1, CL>();
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cfg;
}

// Clusters of CL that can be resident at once on this device (0 if none).
template <int CAP, int CL>
int split_clusters(const q4::DeviceInfo &dev) {
    static q4::DeviceValue cached;
    return cached.get(dev.device, [&] {
        int n = 0;
        if (configure<1, CAP, CL>(dev) == cudaSuccess) {
            cudaLaunchAttribute attr[2];
            cudaLaunchConfig_t cfg = cluster_config<CL>(std::max(1, dev.sm_count / CL), nullptr, attr);
            if (cudaOccupancyMaxActiveClusters(&n, decode_mma_kernel<1, CAP, CL>, &cfg) != cudaSuccess) n = 0;
        }
        (void)cudaGetLastError();
        return std::max(0, std::min(n, kMaxSplitCtas / CL));
    });
}

template <int CAP>
int split_clusters(const q4::DeviceInfo &dev, int cl) {
    switch (cl) {
        case 2: return split_clusters<CAP, 2>(dev);
        case 4: return split_clusters<CAP, 4>(dev);
        case 6: return split_clusters<CAP, 6>(dev);
        case 8: return split_clusters<CAP, 8>(dev);
        default: return 0;
    }
}

// How an M <= 8 launch runs: plain (cl = 1) or in clusters of cl.
struct SplitPlan {
    int cl = 1, clusters = 0;
};

// Launches with at least one item per SM (up to kMaxItems) run in pairs: the
// long items of a decoder layer are halved, the rest stay whole.  Launches
// with fewer items than SMs leave most SMs idle in plain mode; there every
// item can be cut into CL = 4, 6 or 8 pieces on the CTAs of one cluster,
// and the cluster size with the least work on the busiest CTA is taken,
// counting one stage for the hand-over of the partial sums, if that beats
// one whole item per CTA.
constexpr long kHandOverStages = 1;

template <int CAP>
SplitPlan choose_plan(DecodeParams<CAP> &D, const q4::DeviceInfo &dev) {
    const GroupParams<CAP> &P = D.g;
    SplitPlan best;
    if (P.total_items > kMaxItems) return best;
    static thread_local std::vector<q4split::PlanProblem> pp;
    static thread_local q4split::Schedule sc, best_sc;
    pp.resize(P.count);
    for (int i = 0; i < P.count; ++i)
        pp[i] = {P.p[i].stages, P.p[i].item_begin,
                 (i + 1 < P.count ? P.p[i + 1].item_begin : P.total_items) - P.p[i].item_begin};
    if (P.total_items >= dev.sm_count) {
        const int clusters = std::min(split_clusters<CAP>(dev, 2), P.total_items);
        if (clusters < 1) return best;
        q4split::plan(pp.data(), P.count, clusters, 2, sc);
        if (sc.entries > kMaxSched) return best;
        best = {2, clusters};
        q4split::write(sc, clusters, 2, D.sched_begin, D.sched);
        return best;
    }
    long best_cost = 0;
    for (int i = 0; i < P.count; ++i) best_cost = std::max<long>(best_cost, P.p[i].stages);
    for (int cl : {4, 6, 8}) {
        const int clusters = std::min(split_clusters<CAP>(dev, cl), P.total_items);
        if (clusters < 1) continue;
        q4split::plan(pp.data(), P.count, clusters, cl, sc);
        if (sc.entries > kMaxSched) continue;
        const long cost = sc.max_load + kHandOverStages;
        if (cost < best_cost) {
            best_cost = cost;
            best = {cl, clusters};
            std::swap(best_sc, sc);
        }
    }
    if (best.cl > 1) q4split::write(best_sc, best.clusters, best.cl, D.sched_begin, D.sched);
    return best;
}

template <int CAP, int CL>
cudaError_t launch_cluster(const DecodeParams<CAP> &D, int clusters, cudaStream_t s) {
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = cluster_config<CL>(clusters, s, attr);
    return cudaLaunchKernelEx(&cfg, decode_mma_kernel<1, CAP, CL>, D);
}

// The plan and schedule depend only on the device and on each problem's
// stages and item count; a call with the same shapes as the previous one on
// this thread (the usual case: the same layer every token) keeps the
// schedule that `D` still holds.
template <int CAP>
cudaError_t launch_m8(DecodeParams<CAP> &D, const q4::DeviceInfo &dev, cudaStream_t s) {
    static thread_local std::vector<int> last;
    static thread_local SplitPlan plan;
    thread_local std::vector<int> sig;
    const GroupParams<CAP> &P = D.g;
    sig.assign({dev.device, P.count, P.total_items});
    for (int i = 0; i < P.count; ++i) {
        sig.push_back(P.p[i].stages);
        sig.push_back(P.p[i].item_begin);
    }
    if (sig != last) {
        plan = choose_plan(D, dev);
        last = sig;
    }
    switch (plan.cl) {
        case 2: return launch_cluster<CAP, 2>(D, plan.clusters, s);
        case 4: return launch_cluster<CAP, 4>(D, plan.clusters, s);
        case 6: return launch_cluster<CAP, 6>(D, plan.clusters, s);
        case 8: return launch_cluster<CAP, 8>(D, plan.clusters, s);
        default: return launch_plain<1, CAP>(D, dev, s);
    }
}

// problems[order[0..count)] sorted by K (largest first), count <= CAP
template <int CAP>
cudaError_t launch_cap(const q4::Problem *probs, const int *order, int count, const q4::DeviceInfo &dev,
                       cudaStream_t s) {
    static thread_local DecodeParams<CAP> D;
    GroupParams<CAP> &P = D.g;
    P.count = count;
    P.err = dev.err;
    int items = 0;
    int64_t maxM = 1;
    for (int i = 0; i < count; ++i) {
        const q4::Problem &q = probs[order[i]];
        GroupProblem &t = P.p[i];
        t.W = q.W;
        t.X = q.X;
        t.Y = q.Y;
        t.R = q.R;
        t.epi = q.epi;
        t.M = static_cast<int>(q.M);
        t.N = static_cast<int>(q.N);
        t.K = static_cast<int>(q.K);
        t.stages = static_cast<int>(q.K / kStageK);
        t.item_begin = items;
        items += static_cast<int>((q.N + kItemRows - 1) / kItemRows);
        maxM = std::max(maxM, q.M);
        if (!q4::get_tensor_map(&P.wmap[i], q.W, q.N, q.K / 32 * 18, q4::kMapWeights128))
            return cudaErrorInvalidValue;
    }
    P.total_items = items;
    if (maxM > 8) {
        if constexpr (CAP <= kXMapCap) {
            for (int i = 0; i < count; ++i) {
                const q4::Problem &q = probs[order[i]];
                if (!q4::get_tensor_map(&D.xmap[i], q.X, q.M, q.K, maxM <= 16 ? q4::kMapXDecode16 : q4::kMapXDecode32))
                    return cudaErrorInvalidValue;
            }
            if (maxM <= 16) return launch_plain<2, CAP>(D, dev, s);
            return launch_plain<4, CAP>(D, dev, s);
        } else {
            return cudaErrorInvalidValue;   // the caller sends M > 8 groups in chunks of kXMapCap
        }
    }
    return launch_m8<CAP>(D, dev, s);
}

constexpr int kSmallCap = 8, kLargeCap = 128;

}  // namespace

namespace q4 {

bool decode_mma_supports(const Problem &p) {
    return p.M >= 1 && p.M <= 32 && p.K >= kStageK && p.K % kStageK == 0 && p.N >= 1 && p.N < (1LL << 31) &&
           p.K < (1LL << 31) && (reinterpret_cast<uintptr_t>(p.W) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(p.X) & 15) == 0 && tensor_maps_available();
}

cudaError_t launch_decode_mma(const Problem *probs, int count, const DeviceInfo &dev, cudaStream_t s) {
    if (count <= 0) return cudaSuccess;
    static thread_local std::vector<int> order;
    order.resize(count);
    for (int i = 0; i < count; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return probs[a].K > probs[b].K; });
    int64_t maxM = 1;
    for (int i = 0; i < count; ++i) maxM = std::max(maxM, probs[i].M);
    const int cap = maxM > 8 ? kXMapCap : kLargeCap;   // X maps for M > 8 take parameter space
    for (int done = 0; done < count;) {
        const int n = std::min(count - done, cap);
        cudaError_t e = n <= kSmallCap ? launch_cap<kSmallCap>(probs, order.data() + done, n, dev, s)
                        : cap == kXMapCap ? launch_cap<kXMapCap>(probs, order.data() + done, n, dev, s)
                                          : launch_cap<kLargeCap>(probs, order.data() + done, n, dev, s);
        if (e != cudaSuccess) return e;
        done += n;
    }
    return cudaSuccess;
}

}  // namespace q4
