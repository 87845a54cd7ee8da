// q4_0_decode_m8.cu -- the memory-bound decode path for M <= 8 (one token
// step of one or a few sequences: the M = 1 GEMV, batch-2 CFG): one
// persistent launch streams the Q4_0 weights of one or many problems once
// from HBM, dequantizes them in registers and multiplies them with the few
// activation rows on the warp-level tensor cores (mma.sync m16n8k16).
//
// The pages' token loop runs a Q4 matmul for every decoder linear of each of
// the 26 layers (voxtral-mini-realtime-rs (Shannon-Prime fork) README,
// "Architecture Summary"; decode is most of the time: "Pipeline Overlap"),
// with batch-2 CFG and fused QKV / gate-up projections ("TTS
// (Text-to-Speech)", optimizations).
//
// At HBM speed an SM has about 25 warp-instruction slots per 8 weights of a
// lane (6.5 TB/s of 4.5-bit weights over 148 SMs at 1.965 GHz, four issue
// slots per cycle).  The dequantization and the MMA take about 15 of them
// (mask-or into the fp16 pattern of 1024, one packed subtract, one packed
// multiply by d per pair of weights, one MMA per 8 weights of a lane), so this
// kernel is written to spend as little as possible on everything else:
//  * a ring slot holds two 256-k stages (512 k) of a 128-row item: two TMA
//    boxes of 128 rows x 144 bytes plus the stage's X rows (1-D bulk copies),
//    so every wait, arrival and address step covers 512 k;
//  * two groups of 8 compute warps take alternate slots; each warp walks only
//    its own slots, with its ring position and barrier phases kept as
//    counters (no division per slot) and all addresses 32-bit shared-space
//    offsets from one per-thread base;
//  * compute warp w of a group owns rows 16w .. 16w+15; thread (g, t) loads
//    the 36 contiguous bytes of blocks 2t and 2t+1 of rows g and g+8 (nine
//    conflict-free 4-byte loads per row and stage), turns them into fp16
//    (q - 8) * d pairs and feeds them as A fragments of 16 mma.sync per stage:
//    with the scale folded into each weight, one MMA may mix blocks, so every
//    byte a thread loads is its own;
//  * the compute warps also convert the slot's X rows to fp16, straight into
//    the MMA's B fragments: each takes a share of the (stage, X row) pairs,
//    only the M real rows, one 16-byte chunk per lane, and arrives on the
//    group's fragment barrier before it computes (a separate conversion warp
//    got only a fair share of its scheduler's issue slots and could never run
//    ahead, so compute warps waited on it); the fragments are stored as pairs
//    so that a compute thread fetches the two fragments of a code word with
//    one 16-byte load;
//  * the accumulators (two chains) live across the whole item; at its end the
//    group that worked the item's last slot stores Y (optionally + R, or
//    silu(gate) * up), the other group's warps handing their sums over
//    through a double-buffered exchange without waiting.
// Split mode (up to q4split::kMaxItems items): launches of few items leave a
// tail or idle SMs, so the CTAs run in clusters of CL (2 when there is at
// least one item per SM, else 4, 6 or 8); items longer than the mean load of
// a CTA are cut into CL pieces, one per CTA of a cluster, and ranks 1..CL-1
// hand their sums to rank 0 through distributed shared memory (rank 0 adds
// them in rank order, so the result does not depend on timing).
// Launches use programmatic stream serialization: the next grid on the
// stream may start as this grid's CTAs leave; every CTA waits for the
// previous grid before it reads anything into the SM.
// Numerics: each weight is rounded once to fp16 (relative error <= 2^-11,
// inside the 1e-3 tolerance of the method); X is exact in fp16 within its
// normal range; products are exact and accumulation is fp32.  An X too large
// for fp16 (checked once per problem) or a scale that makes a weight overflow
// (looked for when a row's sum is not finite) sets Q4_DEVERR_FP16_RANGE.
// A slot read with ordinary loads is released with a proxy fence first, so
// the next TMA copy into it cannot land before those loads have read it.
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

constexpr int kSub = 2;                               // 256-k stages per ring slot
constexpr int kRawW = kItemRows * kStageRowBytes;     // 18432: one stage of 128 weight rows
constexpr int kXPitch = 512;                          // X row pitch: lanes read 16-byte chunks of one row at a time
constexpr int kSubBytes = kRawW + 8 * kXPitch;        // 22528 (a multiple of 128)
constexpr int kSlotBytes = kSub * kSubBytes;          // 45056
constexpr int kXBufs = 4;                             // fragment buffers: group G uses G and G + 2

constexpr int kWarpProd = 0, kWarp0 = 1, kGroupWarps = 8;
constexpr int kThreads = 32 * (kWarp0 + 2 * kGroupWarps);   // 544
static_assert(kSubBytes % 128 == 0 && kXPitch % 16 == 0, "TMA and bulk-copy destinations stay aligned");

using q4split::kMaxItems;
using q4split::kMaxSched;
using q4split::kMaxSplitCtas;
using q4split::kSplitFlag;

// Ring slots: clusters of 4 and more (launches of few items, where a CTA
// works a few stages) give part of the ring to the partner sums.
template <int CL> constexpr int ring() { return CL >= 6 ? 2 : CL == 4 ? 3 : 4; }

// Partner sums in split mode: rank r > 0 of a cluster of CL writes its sums
// remotely into slot r - 1 of rank 0's copy (two buffers, by item parity).
template <int CL>
struct PartnerSums {
    float v[2][CL - 1][8][4][32];
    uint64_t full[2], empty[2];
};
template <>
struct PartnerSums<1> {};

template <int CL>
struct Smem {
    uint8_t raw[ring<CL>()][kSub][kSubBytes];   // per stage: W rows (pitch 144), then X rows (pitch 512)
    uint4 frag[kXBufs][kSub][8][32];            // B fragment pairs: [buffer][stage][pair][lane]
    float comb[2][8][4][32];                    // an item's sums handed to the group that stores it (by item parity)
    float epi[4][4][32];                        // SwiGLU: up-row sums handed to the gate rows
    uint64_t raw_full[ring<CL>()], raw_empty[ring<CL>()];
    uint64_t frag_full[kXBufs];
    uint64_t comb_full[2], comb_empty[2], epi_full, epi_empty;
    PartnerSums<CL> x;
    int abort_flag;
};

template <int CL>
constexpr size_t smem_bytes() { return sizeof(Smem<CL>) + 128; }
static_assert(smem_bytes<1>() <= 232448, "shared memory budget");
static_assert(smem_bytes<2>() <= 232448, "shared memory budget");
static_assert(smem_bytes<4>() <= 232448, "shared memory budget");
static_assert(smem_bytes<6>() <= 232448, "shared memory budget");
static_assert(smem_bytes<8>() <= 232448, "shared memory budget");

template <int CAP>
struct M8Params {
    GroupParams<CAP> g;
    // split mode: CTA b runs sched[sched_begin[b] .. sched_begin[b+1]), each
    // entry an item index, with kSplitFlag set for a piece of a split item
    uint16_t sched_begin[kMaxSplitCtas + 1];
    uint16_t sched[kMaxSched];
};

// ---------------------------------------------------------------- small device helpers

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

__device__ __forceinline__ void sts64(uint32_t a, uint32_t x, uint32_t y) {
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(a), "r"(x), "r"(y) : "memory");
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

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

// A ring position: slot index and the parity of the barrier phase it is in.
// `step` slots at a time (1 for the producer, 2 for a group's warps).
template <int RS>
struct RingPos {
    int slot;
    uint32_t phase;
    __device__ __forceinline__ void advance(int step) {
        slot += step;
        if (slot >= RS) {   // step <= RS: at most one wrap
            slot -= RS;
            phase ^= 1u;
        }
    }
};

// ---------------------------------------------------------------- the walk over items

// One CTA's items.  Plain mode (CL = 1): items dealt to the CTAs in
// boustrophedon order (round r hands item r*G + b to CTA b when r is even
// and to CTA G-1-b when r is odd), so a CTA's items rise and the problem of
// each is found by a forward scan.  Split mode: the CTA's list from the host;
// of a split n-stage item rank r of the cluster of CL takes stages
// ceil(n r / CL) .. ceil(n (r + 1) / CL) - 1.
template <int CL>
struct Items {
    int round = 0, idx = -1, prob = 0;
    int row0 = 0, s0 = 0, s1 = 0;   // this item: rows row0.., stages [s0, s1)
    bool split = false;

    template <int CAP>
    __device__ __forceinline__ bool next(const M8Params<CAP> &D, uint32_t rank) {
        const GroupParams<CAP> &P = D.g;
        int item;
        if constexpr (CL == 1) {
            const int G = gridDim.x;
            const int pos = (round & 1) ? (G - 1 - static_cast<int>(blockIdx.x)) : static_cast<int>(blockIdx.x);
            item = round * G + pos;
            ++round;
            if (item >= P.total_items) return false;
            while (prob + 1 < P.count && P.p[prob + 1].item_begin <= item) ++prob;
            s0 = 0;
            s1 = P.p[prob].stages;
            split = false;
        } else {
            if (idx < 0) idx = D.sched_begin[blockIdx.x];
            if (idx >= D.sched_begin[blockIdx.x + 1]) return false;
            const uint16_t e = D.sched[idx++];
            item = e & (kSplitFlag - 1);
            split = (e & kSplitFlag) != 0;
            prob = find_problem(P, item);
            const int n = P.p[prob].stages;
            s0 = split ? q4split::piece_begin(n, static_cast<int>(rank), CL) : 0;
            s1 = split ? q4split::piece_begin(n, static_cast<int>(rank) + 1, CL) : n;
        }
        row0 = (item - P.p[prob].item_begin) * kItemRows;
        return true;
    }
};

// ---------------------------------------------------------------- dequantization + MMA

// Rows g and g+8 of one stage: 9 words each (blocks 2t and 2t+1 of the row).
// MMAs (B, W) of the stage: code word W of block 2t+B, low nibbles into
// acc[0], high nibbles into acc[1].
template <int B, int W>
__device__ __forceinline__ void word_mma(const uint32_t (&r)[9], const uint32_t (&r8)[9], uint4 f,
                                         float (&acc)[2][4]) {
    uint32_t dg, dg8, vg, vg8;
    if constexpr (B == 0) {   // block 2t starts 4-byte aligned: d = low half of r[0], codes straddle words
        dg = prmt(r[0], r[0], 0x1010u);
        dg8 = prmt(r8[0], r8[0], 0x1010u);
        vg = prmt(r[W], r[W + 1], 0x5432u);
        vg8 = prmt(r8[W], r8[W + 1], 0x5432u);
    } else {                  // block 2t+1 starts at 2 mod 4: d = high half of r[4], codes aligned
        dg = prmt(r[4], r[4], 0x3232u);
        dg8 = prmt(r8[4], r8[4], 0x3232u);
        vg = r[5 + W];
        vg8 = r8[5 + W];
    }
    uint32_t cg[4], cg8[4];
    q4_word_to_fp16(vg, dg, cg);
    q4_word_to_fp16(vg8, dg8, cg8);
    // a0/a1: k slots (2t, 2t+1) of rows g / g+8; a2/a3: k slots (2t+8, 2t+9)
    mma_f16(acc[0], cg[0], cg8[0], cg[1], cg8[1], f.x, f.y);
    mma_f16(acc[1], cg[2], cg8[2], cg[3], cg8[3], f.z, f.w);
}

// This thread's words of one stage: rows g and g+8 (`w` = shared address of
// the row-g words).
__device__ __forceinline__ void stage_words(uint32_t w, uint32_t (&r)[9], uint32_t (&r8)[9]) {
    #pragma unroll
    for (int i = 0; i < 9; ++i) {
        r[i] = lds32(w + 4 * i);
        r8[i] = lds32(w + 8 * kStageRowBytes + 4 * i);
    }
}

// The 16 MMAs of one stage: `fa` = shared address of this lane's fragment
// pair 0.
__device__ __forceinline__ void stage_mma(const uint32_t (&r)[9], const uint32_t (&r8)[9], uint32_t fa,
                                          float (&acc)[2][4]) {
    word_mma<0, 0>(r, r8, lds128(fa + 0 * 512), acc);
    word_mma<0, 1>(r, r8, lds128(fa + 1 * 512), acc);
    word_mma<0, 2>(r, r8, lds128(fa + 2 * 512), acc);
    word_mma<0, 3>(r, r8, lds128(fa + 3 * 512), acc);
    word_mma<1, 0>(r, r8, lds128(fa + 4 * 512), acc);
    word_mma<1, 1>(r, r8, lds128(fa + 5 * 512), acc);
    word_mma<1, 2>(r, r8, lds128(fa + 6 * 512), acc);
    word_mma<1, 3>(r, r8, lds128(fa + 7 * 512), acc);
}

// ---------------------------------------------------------------- the kernel

template <int CAP, int CL>
__global__ void __launch_bounds__(kThreads, 1) decode_m8_kernel(const __grid_constant__ M8Params<CAP> D) {
    constexpr int RS = ring<CL>();
    const GroupParams<CAP> &P = D.g;
    extern __shared__ uint8_t smem_raw[];
    using SM = Smem<CL>;
    SM &S = *reinterpret_cast<SM *>(align_smem<128>(smem_raw));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t raw0 = smem_addr(&S.raw[0][0][0]);
    const uint32_t frag0 = smem_addr(&S.frag[0][0][0][0]);

    if (threadIdx.x == 0) {
        for (int s = 0; s < RS; ++s) {
            mbar_init(&S.raw_full[s], 1);
            mbar_init(&S.raw_empty[s], kGroupWarps);
        }
        for (int s = 0; s < kXBufs; ++s) mbar_init(&S.frag_full[s], kGroupWarps);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&S.comb_full[s], kGroupWarps);
            mbar_init(&S.comb_empty[s], kGroupWarps);
        }
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
    // into the SM before the previous kernel on the stream has completed.
    // Before that wait the producer only asks L2 for the weight tiles of the
    // CTA's first ring of slots: L2 is where every SM's writes land, so a
    // tile the previous kernel still writes is current when this grid reads it.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == kWarpProd && lane == 0) {
        Items<CL> it;
        int stages = 0, prob = -1;
        while (stages < RS * kSub && it.next(D, rank)) {
            if (it.prob != prob) prefetch_tensormap(&P.wmap[it.prob]);
            prob = it.prob;
            for (int s = it.s0; s < it.s1 && stages < RS * kSub; ++s, ++stages)
                tma_prefetch_l2_2d(&P.wmap[it.prob], s * kStageRowBytes, it.row0);
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    uint32_t prod_issued = 0;

    if (warp == kWarpProd) {
        // ---------------------------------------------------------------- loads
        // every slot in order: wait until both groups' readers released it,
        // then the two weight boxes and the X rows of its two stages
        Items<CL> it;
        RingPos<RS> rp{0, 0};
        bool ok = true;
        while (ok && it.next(D, rank)) {
            const GroupProblem &pr = P.p[it.prob];
            for (int s = it.s0; s < it.s1; s += kSub) {
                const int cnt = min(kSub, it.s1 - s);
                if (lane == 0) ok = wait_or_abort(&S.raw_empty[rp.slot], rp.phase ^ 1u, &S.abort_flag, P.err);
                if (!__shfl_sync(0xffffffffu, ok, 0)) { ok = false; break; }
                if (Q4_DEBUG_BAD(rp.slot >= 0 && rp.slot < RS && cnt >= 1 && cnt <= kSub && pr.M >= 1 && pr.M <= 8,
                                 P.err, &S.abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t dst = raw0 + rp.slot * kSlotBytes;
                if (lane == 0) {
                    // full boxes are counted, zero-filled rows past N included
                    mbar_arrive_expect_tx(&S.raw_full[rp.slot], cnt * (kRawW + pr.M * kStageK * 2));
                    for (int i = 0; i < cnt; ++i)
                        tma_load_2d_u32(dst + i * kSubBytes, &P.wmap[it.prob], (s + i) * kStageRowBytes, it.row0,
                                        &S.raw_full[rp.slot]);
                }
                __syncwarp();
                for (int i = 0; i < cnt; ++i)
                    if (lane < pr.M)
                        bulk_g2s_u32(dst + i * kSubBytes + kRawW + lane * kXPitch,
                                     pr.X + static_cast<int64_t>(lane) * pr.K + static_cast<int64_t>(s + i) * kStageK,
                                     kStageK * 2, &S.raw_full[rp.slot]);
                rp.advance(1);
                ++prod_issued;
            }
        }
    } else {
        // ---------------------------------------------------------------- compute
        const int cw = warp - kWarp0;
        const int G = cw >> 3, tile = cw & 7;   // slot parity, rows 16*tile .. 16*tile+15
        const int gq = lane >> 2, t = lane & 3;
        const uint32_t wbase = raw0 + (16 * tile + gq) * kStageRowBytes + 36 * t;
        // X conversion: lane L takes elements 8L .. 8L+7 of a stage row, i.e.
        // chunk c = L & 7 of window tx = L >> 3 (blocks 2tx and 2tx+1); chunk
        // c = 4B + 2h + W/2 holds code words W, W+1 of block 2tx+B, low (h = 0)
        // or high (h = 1) nibble half, which become half h of fragment pairs
        // 4B + W and 4B + W + 1 of B-fragment lane 4m + tx.  Only the M real
        // rows are converted: fragment columns past M feed accumulator columns
        // that are never stored, so whatever they hold is harmless.
        const int cx = lane & 7;
        const uint32_t fl = (4 * (cx >> 2) + 2 * (cx & 1)) * 512 + (lane >> 3) * 16 + ((cx >> 1) & 1) * 8;
        uint32_t xbad = 0;
        float acc[2][4];
        #pragma unroll
        for (int c = 0; c < 2; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.f;
        RingPos<RS> rp{G, 0};
        int k = 0;
        uint32_t g = 0, items_done = 0, split_done = 0, swiglu_done = 0;
        Items<CL> it;
        while (it.next(D, rank)) {
            const int n = (it.s1 - it.s0 + kSub - 1) / kSub;
            const int M = P.p[it.prob].M;
            // every problem's X is range-checked once, by the CTA (or cluster)
            // that works its first item
            const bool check = it.row0 == 0;
            bool ok = true;
            for (int j = (G - static_cast<int>(g)) & 1; j < n; j += 2, ++k, rp.advance(2)) {
                const int cnt = min(kSub, it.s1 - (it.s0 + kSub * j));
                const int xb = G + 2 * (k & 1);
                // the slot, buffer and byte ranges this slot touches stay inside their arrays
                if (Q4_DEBUG_BAD(rp.slot >= 0 && rp.slot < RS && xb >= 0 && xb < kXBufs && cnt >= 1 &&
                                     cnt <= kSub && M >= 1 && M <= 8 &&
                                     wbase + rp.slot * kSlotBytes + (kSub - 1) * kSubBytes + 8 * kStageRowBytes + 36 <=
                                         raw0 + RS * kSlotBytes &&
                                     frag0 + (xb * kSub + kSub - 1) * 4096 + 7 * 512 + lane * 16 + 16 <=
                                         frag0 + kXBufs * kSub * 4096,
                                 P.err, &S.abort_flag)) {
                    ok = false;
                    break;
                }
                if (!(ok = wait_or_abort(&S.raw_full[rp.slot], rp.phase, &S.abort_flag, P.err))) break;
                // this warp's share of the slot's X rows -> fp16 B fragments:
                // (stage, row) pairs tile and tile + 8 of the cnt * M pairs.
                // Buffer xb was last read by the group's slot k - 2; every warp
                // finished that before it arrived on the fragment barrier of
                // slot k - 1, which this warp has passed.
                {
                    const uint32_t xr = raw0 + rp.slot * kSlotBytes + kRawW + lane * 16;
                    const uint32_t fo = frag0 + xb * kSub * 4096 + fl;
                    for (int pi = tile; pi < cnt * M; pi += kGroupWarps) {
                        const int i = pi >= M ? 1 : 0, m = pi - i * M;
                        const uint4 v = lds128(xr + i * kSubBytes + m * kXPitch);
                        if (check) xbad |= x8_fp16_range_bad(v);
                        const uint4 o = x8_to_fp16_permuted(v);
                        sts64(fo + i * 4096 + m * 64, o.x, o.y);
                        sts64(fo + i * 4096 + 512 + m * 64, o.z, o.w);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.frag_full[xb]);
                // the slot's words into registers, then the slot goes back to the
                // producer (a stage that is not part of the item -- cnt = 1 -- is
                // read but not used)
                const uint32_t w = wbase + rp.slot * kSlotBytes;
                uint32_t r[kSub][9], r8[kSub][9];
                #pragma unroll
                for (int i = 0; i < kSub; ++i) stage_words(w + i * kSubBytes, r[i], r8[i]);
                fence_proxy_async_smem();   // the producer's next copies may land in this slot
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.raw_empty[rp.slot]);
                if (!(ok = wait_or_abort(&S.frag_full[xb], (k >> 1) & 1, &S.abort_flag, P.err))) break;
                const uint32_t fa = frag0 + xb * kSub * 4096 + lane * 16;
                stage_mma(r[0], r8[0], fa, acc);
                if (cnt > 1) stage_mma(r[1], r8[1], fa + 4096, acc);
            }
            if (!ok) break;
            // ------------------------------------------------------------ end of the item
            // The group that worked the item's last slot stores it; the other
            // group hands its sums over (buffer by item parity) and goes on.
            const GroupProblem &pr = P.p[it.prob];
            const int last = static_cast<int>((g + n - 1) & 1);
            g += n;
            const int cb = items_done & 1;
            const uint32_t cpar = (items_done >> 1) & 1;
            ++items_done;
            // every warp counts the split and SwiGLU items, whichever group stores them
            const uint32_t split_k = split_done, swiglu_k = swiglu_done;
            if (it.split) ++split_done;
            if (pr.epi == kEpiSwiGLU && (!it.split || rank == 0)) ++swiglu_done;
            if (G != last) {
                if (!wait_or_abort(&S.comb_empty[cb], cpar ^ 1, &S.abort_flag, P.err)) break;
                #pragma unroll
                for (int e = 0; e < 4; ++e) S.comb[cb][tile][e][lane] = acc[0][e] + acc[1][e];
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.comb_full[cb]);
            } else {
                if (!wait_or_abort(&S.comb_full[cb], cpar, &S.abort_flag, P.err)) break;
                float sum[4];
                #pragma unroll
                for (int e = 0; e < 4; ++e) sum[e] = acc[0][e] + acc[1][e] + S.comb[cb][tile][e][lane];
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.comb_empty[cb]);
                if constexpr (CL > 1) {
                    if (it.split) {
                        // ranks 1..CL-1 hand their sums to rank 0 of the cluster, which adds
                        // them in rank order
                        const int xb2 = split_k & 1;
                        const uint32_t xpar = (split_k >> 1) & 1;
                        if (rank != 0) {
                            if (!wait_cluster_or_abort(&S.x.empty[xb2], xpar ^ 1, &S.abort_flag, P.err)) break;
                            #pragma unroll
                            for (int e = 0; e < 4; ++e) st_remote(&S.x.v[xb2][rank - 1][tile][e][lane], 0, sum[e]);
                            mbar_arrive_remote(&S.x.full[xb2], 0);
                        } else {
                            if (!wait_cluster_or_abort(&S.x.full[xb2], xpar, &S.abort_flag, P.err)) break;
                            #pragma unroll
                            for (int r = 0; r < CL - 1; ++r)
                                #pragma unroll
                                for (int e = 0; e < 4; ++e) sum[e] += S.x.v[xb2][r][tile][e][lane];
                            #pragma unroll
                            for (int r = 1; r < CL; ++r) mbar_arrive_remote(&S.x.empty[xb2], r);
                        }
                    }
                }
                // thread holds rows gq / gq+8 of the tile x X rows 2t, 2t+1
                if (!it.split || rank == 0) {
                    // a non-finite sum from finite inputs means an fp16 weight
                    // overflowed: look at the rows' scales (slow path, rare)
                    bool bad_row[2] = {false, false};
                    #pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (2 * t + (e & 1) < pr.M && !(fabsf(sum[e]) <= 3.402823466e38f)) bad_row[e >> 1] = true;
                    #pragma unroll
                    for (int h = 0; h < 2; ++h)
                        if (bad_row[h]) {
                            const int64_t nn = it.row0 + 16 * tile + gq + 8 * h;
                            scan_scales_fp16_range(pr.W, nn, nn + 1, pr.N, pr.K, P.err);
                        }
                }
                if ((!it.split || rank == 0) && pr.epi == kEpiSwiGLU) {
                    // rows 0-63 of the item are gate rows of features row0/2 .. row0/2+63,
                    // rows 64-127 the up rows of the same features: tiles 4-7 hand their
                    // sums to tiles 0-3, which store silu(gate) * up into Y[M, N/2]
                    const uint32_t epar = swiglu_k & 1;
                    if (tile >= 4) {
                        if (!wait_or_abort(&S.epi_empty, epar ^ 1, &S.abort_flag, P.err)) break;
                        #pragma unroll
                        for (int e = 0; e < 4; ++e) S.epi[tile - 4][e][lane] = sum[e];
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&S.epi_full);
                    } else {
                        if (!wait_or_abort(&S.epi_full, epar, &S.abort_flag, P.err)) break;
                        const int F = pr.N >> 1;
                        #pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float gv = sum[e], uv = S.epi[tile][e][lane];
                            const int m = 2 * t + (e & 1);
                            const int f = (it.row0 >> 1) + 16 * tile + gq + ((e & 2) ? 8 : 0);
                            if (m < pr.M) pr.Y[static_cast<int64_t>(m) * F + f] = gv / (1.0f + expf(-gv)) * uv;
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&S.epi_empty);
                    }
                } else if (!it.split || rank == 0) {
                    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int m = 2 * t + (e & 1);
                        const int nn = it.row0 + 16 * tile + gq + ((e & 2) ? 8 : 0);
                        if (m < pr.M && nn < pr.N) {
                            const int64_t o = static_cast<int64_t>(m) * pr.N + nn;
                            pr.Y[o] = pr.epi == kEpiResidual ? sum[e] + pr.R[o] : sum[e];
                        }
                    }
                }
            }
            #pragma unroll
            for (int c = 0; c < 2; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.f;
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

// ---------------------------------------------------------------- one small problem

// A launch of one problem with few rows (a lone GEMV at M <= 8) is short:
// its time is latency, not bandwidth.  Here each CTA takes 16*NR weight rows
// over all of K, requests all of its weights at once (one TMA box of
// 16*NR rows x 144 bytes per 256-k stage, each on its own barrier), and its
// NW warps (16, 24 or 32) split the work into NR row tiles x NW/NR k-groups
// (k-group j takes stages j, j + NW/NR, ...).  X is converted once per CTA into the B
// fragments of every stage.  The k-groups' partial sums meet in shared memory
// and are added in k-group order by the first k-group's warps, which store
// Y.  No clusters, no ring, no hand-over between CTAs.
struct NarrowParams {
    CUtensorMap wmap;     // Q4_0 bytes [N, K/32*18], box 144 x 16*NR
    const uint8_t *W;     // the same bytes (read directly only by the rare scale check)
    const uint16_t *X;
    float *Y;
    const float *R;       // residual (Q4_0_EPI_RESIDUAL)
    unsigned *err;
    int M, N, K, S, epi;  // S = K / 256 stages
};

template <int NR>
constexpr int narrow_rows() { return 16 * NR; }

// Warps of a CTA.  Where 16 would give a k-group (16 / NR of them) more than
// one stage and the CTA's weights are few (at most 24 stage-row-tiles,
// 55 KB), 24 warps give every k-group at most one stage, which halves the
// longest chain of stages that paces such latency-bound launches; 32 when
// M > 4, where the X conversion (S * M rows of 256 k) wants the extra warps.
// Else 16: with one stage per k-group anyway, or with more weights per SM,
// where the stream paces the launch, a larger CTA only adds its own cost.
// Back to back, 3072^2: M = 1 5.15 -> 3.87 us (24 warps; 4.05 with 32),
// M = 2 5.72 -> 4.01 us, M = 8 7.37 -> 5.26 us (32 warps; 5.40 with 24); with
// 16 warps kept: 4096^2 4.84 against 5.02 us and 2368 x 3072 (16 rows a CTA)
// 3.08 against 3.45 us with 32.
constexpr int narrow_warps(int S, int NR, int M) {
    return NR > 0 && S > 16 / NR && S * NR <= 24 ? (M <= 4 ? 24 : 32) : 16;
}

template <int NR, int NW>
constexpr size_t narrow_smem(int S) {
    return static_cast<size_t>(S) * narrow_rows<NR>() * kStageRowBytes   // weight boxes
           + static_cast<size_t>(S) * 4096                               // B fragment pairs per stage
           + static_cast<size_t>(NW) * 4 * 32 * 4                         // partial sums
           + static_cast<size_t>(S) * 8 + 16 + 128;                      // barriers, abort flag, alignment
}

template <int NR, int NW>
__global__ void __launch_bounds__(32 * NW, 1) narrow_kernel(const __grid_constant__ NarrowParams P) {
    constexpr int KG = NW / NR, ROWS = narrow_rows<NR>();
    constexpr int kBox = ROWS * kStageRowBytes;
    const int S = P.S;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *const wsm = align_smem<128>(smem_raw);
    uint8_t *const fsm = wsm + S * kBox;                                    // kBox is a multiple of 16
    float *const red = reinterpret_cast<float *>(fsm + S * 4096);
    uint64_t *const bar = reinterpret_cast<uint64_t *>(red + NW * 4 * 32);
    int *const abort_flag = reinterpret_cast<int *>(bar + S);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row0 = blockIdx.x * ROWS;
    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) mbar_init(&bar[st], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // programmatic dependent launch: the weights and X are asked into L2
    // before the previous grid is waited for, everything is read after it
    // (CTA m < M asks for row m of X)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        prefetch_tensormap(&P.wmap);
        for (int st = 0; st < S; ++st) tma_prefetch_l2_2d(&P.wmap, st * kStageRowBytes, row0);
    } else if (threadIdx.x == 32 && static_cast<int>(blockIdx.x) < P.M) {
        bulk_prefetch_l2(P.X + static_cast<int64_t>(blockIdx.x) * P.K, static_cast<uint32_t>(P.K * 2));
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_arrive_expect_tx(&bar[st], kBox);   // full boxes counted, rows past N zero-filled
            tma_load_2d_u32(smem_addr(wsm + st * kBox), &P.wmap, st * kStageRowBytes, row0, &bar[st]);
        }
    }
    // X -> fp16 B fragments of every stage: the (stage, row) pairs dealt over
    // the warps, one 16-byte chunk (8 values) per lane, in the layout the
    // decode kernel's stage_mma reads
    const uint32_t f0 = smem_addr(fsm);
    uint32_t xbad = 0;
    {
        const int cx = lane & 7;
        const uint32_t fl = (4 * (cx >> 2) + 2 * (cx & 1)) * 512 + (lane >> 3) * 16 + ((cx >> 1) & 1) * 8;
        for (int pi = warp; pi < S * P.M; pi += NW) {
            const int st = pi / P.M, m = pi - st * P.M;
            if (Q4_DEBUG_BAD(st < S && m < P.M, P.err, abort_flag)) break;
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(P.X + static_cast<int64_t>(m) * P.K + st * kStageK) +
                                  lane);
            if (blockIdx.x == 0) xbad |= x8_fp16_range_bad(v);   // every row of X checked once
            const uint4 o = x8_to_fp16_permuted(v);
            sts64(f0 + st * 4096 + fl + m * 64, o.x, o.y);
            sts64(f0 + st * 4096 + fl + 512 + m * 64, o.z, o.w);
        }
    }
    __syncthreads();
    // this warp's row tile and k-group
    const int rt = warp % NR, kg = warp / NR;
    const int gq = lane >> 2, t = lane & 3;
    float acc[2][4];
    #pragma unroll
    for (int c = 0; c < 2; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.f;
    const uint32_t w0 = smem_addr(wsm) + (16 * rt + gq) * kStageRowBytes + 36 * t;
    bool ok = true;
    for (int st = kg; st < S; st += KG) {
        if (!(ok = wait_or_abort(&bar[st], 0, abort_flag, P.err))) break;
        uint32_t r[9], r8[9];
        stage_words(w0 + st * kBox, r, r8);
        stage_mma(r, r8, f0 + st * 4096 + lane * 16, acc);
    }
    {
        float *const mine = red + ((rt * KG + kg) * 4) * 32;
        #pragma unroll
        for (int e = 0; e < 4; ++e) mine[e * 32 + lane] = acc[0][e] + acc[1][e];
    }
    __syncthreads();
    if (kg == 0 && ok && !*reinterpret_cast<volatile int *>(abort_flag)) {
        float sum[4] = {0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < KG; ++j) {
            const float *part = red + ((rt * KG + j) * 4) * 32;
            #pragma unroll
            for (int e = 0; e < 4; ++e) sum[e] += part[e * 32 + lane];
        }
        // thread holds rows gq / gq+8 of the row tile x X rows 2t, 2t+1
        bool bad_row[2] = {false, false};
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int m = 2 * t + (e & 1);
            const int n = row0 + 16 * rt + gq + ((e & 2) ? 8 : 0);
            if (m < P.M && n < P.N) {
                if (!(fabsf(sum[e]) <= 3.402823466e38f)) bad_row[e >> 1] = true;
                const int64_t o = static_cast<int64_t>(m) * P.N + n;
                P.Y[o] = P.epi == kEpiResidual ? sum[e] + P.R[o] : sum[e];
            }
        }
        #pragma unroll
        for (int h = 0; h < 2; ++h)
            if (bad_row[h]) {
                const int64_t n = row0 + 16 * rt + gq + 8 * h;
                scan_scales_fp16_range(P.W, n, n + 1, P.N, P.K, P.err);
            }
    }
    if (xbad) atomicOr(P.err, (unsigned)Q4_DEVERR_FP16_RANGE);
    // a wait that gave up: let every box land (bounded) before the CTA exits
    if (threadIdx.x == 0 && *reinterpret_cast<volatile int *>(abort_flag))
        for (int st = 0; st < S; ++st) mbar_wait(&bar[st], 0, P.err);
}

// ---------------------------------------------------------------- host side

template <int CAP, int CL>
cudaError_t configure(const q4::DeviceInfo &dev) {
    static q4::DeviceOnce configured;
    return configured.run(dev.device, [] {
        return cudaFuncSetAttribute(decode_m8_kernel<CAP, CL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem_bytes<CL>()));
    });
}

template <int CL>
cudaLaunchConfig_t launch_config(int ctas, cudaStream_t s, cudaLaunchAttribute *attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ctas, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes<CL>();
    cfg.stream = s;
    int n = 0;
    if constexpr (CL > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = CL;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cfg;
}

template <int CAP, int CL>
cudaError_t launch(const M8Params<CAP> &D, int ctas, const q4::DeviceInfo &dev, cudaStream_t s) {
    cudaError_t e = configure<CAP, CL>(dev);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = launch_config<CL>(ctas, s, attr);
    return cudaLaunchKernelEx(&cfg, decode_m8_kernel<CAP, CL>, D);
}

// Clusters of CL that can be resident at once on this device (0 if none).
template <int CAP, int CL>
int resident_clusters(const q4::DeviceInfo &dev) {
    static q4::DeviceValue cached;
    return cached.get(dev.device, [&] {
        int n = 0;
        if (configure<CAP, CL>(dev) == cudaSuccess) {
            cudaLaunchAttribute attr[2];
            cudaLaunchConfig_t cfg = launch_config<CL>(CL * std::max(1, dev.sm_count / CL), nullptr, attr);
            if (cudaOccupancyMaxActiveClusters(&n, decode_m8_kernel<CAP, CL>, &cfg) != cudaSuccess) n = 0;
        }
        (void)cudaGetLastError();
        return std::max(0, std::min(n, kMaxSplitCtas / CL));
    });
}

template <int CAP>
int resident_clusters(const q4::DeviceInfo &dev, int cl) {
    switch (cl) {
        case 2: return resident_clusters<CAP, 2>(dev);
        case 4: return resident_clusters<CAP, 4>(dev);
        case 6: return resident_clusters<CAP, 6>(dev);
        case 8: return resident_clusters<CAP, 8>(dev);
        default: return 0;
    }
}

// How a launch runs: plain (cl = 1) or in clusters of cl.
struct SplitPlan {
    int cl = 1, clusters = 0;
};

// Launches with at least one item per SM (up to kMaxItems) run in pairs: the
// long items of a decoder layer are halved, the rest stay whole.  Launches
// with fewer items than SMs leave most SMs idle in plain mode; there every
// item can be cut into CL = 4, 6 or 8 pieces on the CTAs of one cluster, and
// the cluster size with the least work on the busiest CTA is taken, counting
// one stage for the hand-over of the partial sums, if that beats one whole
// item per CTA.
constexpr long kHandOverStages = 1;

template <int CAP>
SplitPlan choose_plan(M8Params<CAP> &D, const q4::DeviceInfo &dev) {
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
        const int clusters = std::min(resident_clusters<CAP>(dev, 2), P.total_items);
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
        const int clusters = std::min(resident_clusters<CAP>(dev, cl), P.total_items);
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

// problems[order[0..count)] sorted by K (largest first), count <= CAP.  The
// plan and schedule depend only on the device and on each problem's stages
// and item count; a call with the same shapes as the previous one on this
// thread (the usual case: the same layer every token) keeps the schedule
// that `D` still holds.
template <int CAP>
cudaError_t launch_cap(const q4::Problem *probs, const int *order, int count, const q4::DeviceInfo &dev,
                       cudaStream_t s) {
    static thread_local M8Params<CAP> D;
    static thread_local std::vector<int> last;
    static thread_local SplitPlan plan;
    static thread_local std::vector<int> sig;
    GroupParams<CAP> &P = D.g;
    P.count = count;
    P.err = dev.err;
    int items = 0;
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
        if (!q4::get_tensor_map(&P.wmap[i], q.W, q.N, q.K / 32 * 18, q4::kMapWeights128))
            return cudaErrorInvalidValue;
    }
    P.total_items = items;
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
        case 2: return launch<CAP, 2>(D, 2 * plan.clusters, dev, s);
        case 4: return launch<CAP, 4>(D, 4 * plan.clusters, dev, s);
        case 6: return launch<CAP, 6>(D, 6 * plan.clusters, dev, s);
        case 8: return launch<CAP, 8>(D, 8 * plan.clusters, dev, s);
        default: return launch<CAP, 1>(D, std::max(1, std::min(dev.sm_count, P.total_items)), dev, s);
    }
}

constexpr int kSmallCap = 8, kLargeCap = 128;

// The one-problem kernel: 16 or 32 rows per CTA, as many CTAs as that takes,
// when they fit on the SMs at once and the CTA's weights, fragments and sums
// fit in shared memory.  Returns the row tiles per CTA (1 or 2), 0 if not.
int narrow_rows_per_cta(const q4::Problem &p, const q4::DeviceInfo &dev) {
    if (p.M < 1 || p.M > 8 || p.K < kStageK || p.K % kStageK != 0 || p.N < 1) return 0;
    if (p.epi != kEpiNone && p.epi != kEpiResidual) return 0;
    const int S = static_cast<int>(p.K / kStageK);
    const int nr = p.N <= 16LL * dev.sm_count ? 1 : p.N <= 32LL * dev.sm_count ? 2 : 0;
    if (nr == 0) return 0;
    const int nw = narrow_warps(S, nr, static_cast<int>(p.M));
    const size_t smem = nw == 32   ? (nr == 1 ? narrow_smem<1, 32>(S) : narrow_smem<2, 32>(S))
                        : nw == 24 ? (nr == 1 ? narrow_smem<1, 24>(S) : narrow_smem<2, 24>(S))
                                   : (nr == 1 ? narrow_smem<1, 16>(S) : narrow_smem<2, 16>(S));
    return smem <= dev.smem_optin ? nr : 0;
}

template <int NR, int NW>
cudaError_t launch_narrow(const q4::Problem &p, const q4::DeviceInfo &dev, cudaStream_t s) {
    NarrowParams P;
    if (!q4::get_tensor_map(&P.wmap, p.W, p.N, p.K / 32 * 18, NR == 1 ? q4::kMapWeights16 : q4::kMapWeights32))
        return cudaErrorInvalidValue;
    P.W = p.W;
    P.X = p.X;
    P.Y = p.Y;
    P.R = p.R;
    P.err = dev.err;
    P.M = static_cast<int>(p.M);
    P.N = static_cast<int>(p.N);
    P.K = static_cast<int>(p.K);
    P.S = static_cast<int>(p.K / kStageK);
    P.epi = p.epi;
    const size_t smem = narrow_smem<NR, NW>(P.S);
    static q4::DeviceOnce configured;
    cudaError_t e = configured.run(dev.device, [&] {
        return cudaFuncSetAttribute(narrow_kernel<NR, NW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(dev.smem_optin));
    });
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((p.N + narrow_rows<NR>() - 1) / narrow_rows<NR>()), 1, 1);
    cfg.blockDim = dim3(32 * NW, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, narrow_kernel<NR, NW>, P);
}

}  // namespace

namespace q4 {

bool decode_m8_supports(const Problem &p) {
    return p.M >= 1 && p.M <= 8 && p.K >= kStageK && p.K % kStageK == 0 && p.N >= 1 && p.N < (1LL << 31) &&
           p.K < (1LL << 31) && (reinterpret_cast<uintptr_t>(p.W) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(p.X) & 15) == 0 && tensor_maps_available();
}

cudaError_t launch_decode_m8(const Problem *probs, int count, const DeviceInfo &dev, cudaStream_t s) {
    if (count <= 0) return cudaSuccess;
    if (count == 1) {   // a lone small problem: the one-problem kernel
        const int nr = narrow_rows_per_cta(probs[0], dev);
        const int nw = narrow_warps(static_cast<int>(probs[0].K / kStageK), nr, static_cast<int>(probs[0].M));
        if (nr == 1)
            return nw == 32   ? launch_narrow<1, 32>(probs[0], dev, s)
                   : nw == 24 ? launch_narrow<1, 24>(probs[0], dev, s)
                              : launch_narrow<1, 16>(probs[0], dev, s);
        if (nr == 2)
            return nw == 32   ? launch_narrow<2, 32>(probs[0], dev, s)
                   : nw == 24 ? launch_narrow<2, 24>(probs[0], dev, s)
                              : launch_narrow<2, 16>(probs[0], dev, s);
    }
    static thread_local std::vector<int> order;
    order.resize(count);
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
