// q4_0_prefill.cu -- the tensor-core path for M > 32 (prefill, the adapter,
// batched requests): a persistent, warp-specialised tcgen05 kernel.
//
// The pages run the adapter (reshape to width 5120, then 3072) and the
// decoder linears over all prompt/audio frames at once
// (voxtral-mini-realtime-rs (Shannon-Prime fork) README, "Architecture";
// hakusoku.com story 5135, architecture); with thousands of rows of X this
// is a dense contraction, so it belongs on the 5th-generation tensor cores.
//
// Tile: 128 weight rows (n) x 256 activation rows (m), D = W_tile * X_tile^T
// accumulated in fp32 in tensor memory (128 lanes x 256 columns).
//   * A operand = the weight tile, dequantized by four warps straight into
//     tensor memory as fp16 (q - 8) * d: the raw Q4_0 bytes arrive by TMA
//     (128 rows x 144 bytes = 256 k per load), each thread turns its row's
//     blocks into fp16 pairs and writes them with tcgen05.st;
//   * B operand = the activation tile, loaded by TMA into the
//     128-byte-swizzled K-major layout the MMA reads: as fp16 written once by
//     the pre-pass (x_to_fp16_kernel: q4_0_gemm_ws, or q4_0_prepare_x on its
//     own) or as bf16, converted to fp16 in place by eight warps;
//   * one thread issues tcgen05.mma (kind::f16, M=128, N=256, K=16), four per
//     64-k stage, and signals stage release with tcgen05.commit;
//   * four epilogue warps drain the accumulator with tcgen05.ld; lane = weight
//     row, column = activation row, so each store of a column is one
//     contiguous 128-byte run of Y[m, n0..n0+31]; they add a residual or
//     apply SwiGLU on the way (q4_0_gemm_grouped_ex).
// fp16 operands: a weight (q - 8) * d is rounded once to fp16 (relative error
// <= 2^-11, inside the 1e-3 tolerance of the method); X is exact in fp16 in
// the normal range.  Both must lie within the fp16 range (|x| <= 65504,
// |d| <= 8188): beyond it the products overflow to +-inf.  Inside each block
// of 32 the k order is permuted identically for both operands (positions 1
// and 2 of every 4 swapped), which lets the dequantization emit the nibble
// pairs in the order the packed bytes hold them.
#include <cuda.h>
#include <cuda_fp16.h>

#include <cstring>
#include <mutex>

#include "q4_0_internal.cuh"
#include "q4_0_convert.cuh"
#include "q4_0_tcgen05.cuh"
#include "q4_0_tmap.cuh"

namespace {

using namespace q4dev;

constexpr int kTileN = 128;                    // weight rows per tile (MMA M)
constexpr int kTileM = 256;                    // activation rows per tile (MMA N)
constexpr int kStageK = 64;                    // k per operand stage (one 128-byte swizzle row)
constexpr int kRawK = 256;                     // k per raw weight load (8 blocks = 144 bytes)
static_assert(kRawK == 4 * kStageK, "a raw weight load feeds four operand stages");
constexpr int kXStages = 4;
constexpr int kRawStages = 2;
constexpr int kAStages = 4;                    // A buffers in tensor memory
constexpr int kXStageBytes = kTileM * 128;     // 32 KB
constexpr int kRawRowBytes = 144;
constexpr int kRawStageBytes = kTileN * kRawRowBytes;   // 18 KB
constexpr int kTmemCols = 512;
constexpr int kDCol = 0;                       // accumulator columns [0, 256)
constexpr int kACol = 256;                     // A buffers: 32 columns each

constexpr int kWarpTMA = 0, kWarpMMA = 1;
constexpr int kWarpDeq0 = 2, kNumDeq = 4;      // warps 2..5
constexpr int kWarpCvt0 = 6, kNumCvt = 8;      // warps 6..13 (X converted in the kernel)
constexpr int kNumEpi = 4;                     // then 4 epilogue warps
// XPRE: X arrives already in fp16 (converted once by the pre-pass into the
// caller's workspace), so the eight conversion warps are not launched.
template <bool XPRE> constexpr int epi_warp0() { return XPRE ? kWarpCvt0 : kWarpCvt0 + kNumCvt; }
template <bool XPRE> constexpr int threads() { return 32 * (epi_warp0<XPRE>() + kNumEpi); }

struct alignas(64) PrefillParams {
    CUtensorMap tmap_x;    // bf16 [M, K], box 64 x 256, 128-byte swizzle
    CUtensorMap tmap_w;    // uint8 [N, K/32*18], box 144 x 128
    float *Y;
    const uint8_t *W;      // the Q4_0 weights (read directly only by the rare scale check)
    const float *R;        // residual [M, N] (Q4_0_EPI_RESIDUAL; may be Y itself)
    unsigned *err;
    int M, N, K;
    int tiles_n, tiles_m;
    int epi;               // Q4_0_EPI_* (one per launch)
};

struct Smem {
    uint8_t x[kXStages][kXStageBytes];        // 1024-byte aligned (swizzle atoms)
    uint8_t raw[kRawStages][kRawStageBytes];
    uint64_t x_full[kXStages], x_conv[kXStages], x_empty[kXStages];
    uint64_t raw_full[kRawStages], raw_empty[kRawStages];
    uint64_t a_full[kAStages], a_empty[kAStages];
    uint64_t d_full, d_empty, mma_done;
    // SwiGLU epilogue, per 32-column chunk (double-buffered): the up rows'
    // sums of columns 0-15 for the gate rows' warps and the gate rows' sums
    // of columns 16-31 for the up rows' warps, [column][feature of the tile]
    float xch[2][32][64];
    uint64_t xch_full[2], xch_empty[2];
    uint32_t tmem_base;
    int abort_flag;
};

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms of
// 1024 bytes stacked along the row dimension.
__device__ __forceinline__ uint64_t sw128_desc(const void *base) {
    const uint64_t addr = smem_addr(base);
    return ((addr >> 4) & 0x3FFFull) | (1ull << 16) | (uint64_t(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: fp16 x fp16 -> fp32, both K-major, M=128, N=256.
constexpr uint32_t kIdesc = (1u << 4) | (0u << 7) | (0u << 10) | (uint32_t(kTileM >> 3) << 17) |
                            (uint32_t(kTileN >> 4) << 24);

// Bounded wait that also gives up when another role has aborted.
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

// ---------------------------------------------------------------- dequantization

// Block i (0..7) of a 144-byte raw row held in 36 registers: the fp16 scale
// bits and the four qs words.
__device__ __forceinline__ void block_words(const uint32_t (&raw)[36], int i, uint32_t &dbits, uint32_t (&q)[4]) {
    const int b = 18 * i;          // byte offset of the block
    const int w = b >> 2;
    if ((i & 1) == 0) {            // block starts 4-byte aligned: d = low half of raw[w]
        dbits = raw[w] & 0xFFFFu;
        #pragma unroll
        for (int j = 0; j < 4; ++j) q[j] = prmt(raw[w + j], raw[w + j + 1], 0x5432u);
    } else {                       // block starts at 2 mod 4: d = high half, qs aligned
        dbits = raw[w] >> 16;
        #pragma unroll
        for (int j = 0; j < 4; ++j) q[j] = raw[w + 1 + j];
    }
}

// ---------------------------------------------------------------- the kernel

template <bool XPRE>
__global__ void __launch_bounds__(threads<XPRE>(), 1) prefill_kernel(const __grid_constant__ PrefillParams P) {
    extern __shared__ uint8_t smem_raw[];
    Smem &S = *reinterpret_cast<Smem *>(align_smem<1024>(smem_raw));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = P.tiles_n * P.tiles_m;
    const int ksteps = P.K / kStageK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kXStages; ++s) {
            mbar_init(&S.x_full[s], 1);
            mbar_init(&S.x_conv[s], kNumCvt);
            mbar_init(&S.x_empty[s], 1);
        }
        for (int s = 0; s < kRawStages; ++s) {
            mbar_init(&S.raw_full[s], 1);
            mbar_init(&S.raw_empty[s], kNumDeq);
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&S.a_full[s], kNumDeq);
            mbar_init(&S.a_empty[s], 1);
        }
        mbar_init(&S.d_full, 1);
        mbar_init(&S.d_empty, kNumEpi);
        mbar_init(&S.mma_done, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&S.xch_full[b], kNumEpi);
            mbar_init(&S.xch_empty[b], kNumEpi);
        }
        S.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&S.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (warp == kWarpTMA) {
        if (lane == 0) {
            uint32_t xc = 0, rc = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int n0 = (t % P.tiles_n) * kTileN, m0 = (t / P.tiles_n) * kTileM;
                for (int ks = 0; ks < ksteps && ok; ++ks) {
                    if ((ks & 3) == 0) {
                        const int s = rc % kRawStages;
                        if (Q4_DEBUG_BAD(s < kRawStages && n0 < P.tiles_n * kTileN, P.err, &S.abort_flag)) {
                            ok = false;
                            break;
                        }
                        if (!(ok = wait_or_abort(&S.raw_empty[s], ((rc / kRawStages) & 1) ^ 1, S, P.err))) break;
                        mbar_arrive_expect_tx(&S.raw_full[s], kRawStageBytes);
                        tma_load_2d(S.raw[s], &P.tmap_w, (ks >> 2) * kRawRowBytes, n0, &S.raw_full[s]);
                        ++rc;
                    }
                    const int s = xc % kXStages;
                    if (Q4_DEBUG_BAD(s < kXStages && m0 < P.tiles_m * kTileM, P.err, &S.abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (!(ok = wait_or_abort(&S.x_empty[s], ((xc / kXStages) & 1) ^ 1, S, P.err))) break;
                    mbar_arrive_expect_tx(&S.x_full[s], kXStageBytes);
                    tma_load_2d(S.x[s], &P.tmap_x, ks * kStageK, m0, &S.x_full[s]);
                    ++xc;
                }
            }
            if (!ok) {   // let the loads already issued land (bounded) before the CTA can exit
                for (uint32_t i = 0; i < kXStages && i < xc; ++i) {
                    const uint32_t c = xc - 1 - i;
                    mbar_wait(&S.x_full[c % kXStages], (c / kXStages) & 1, P.err);
                }
                for (uint32_t i = 0; i < kRawStages && i < rc; ++i) {
                    const uint32_t c = rc - 1 - i;
                    mbar_wait(&S.raw_full[c % kRawStages], (c / kRawStages) & 1, P.err);
                }
            }
        }
    } else if (warp == kWarpMMA) {
        if (lane == 0) {
            uint32_t xc = 0, ac = 0, dc = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++dc) {
                if (!(ok = wait_or_abort(&S.d_empty, (dc & 1) ^ 1, S, P.err))) break;
                tc_fence_after();
                for (int ks = 0; ks < ksteps; ++ks) {
                    const int sx = xc % kXStages, sa = ac % kAStages;
                    // A buffers and the accumulator stay inside the 512 tensor-memory columns
                    if (Q4_DEBUG_BAD(sx < kXStages && sa < kAStages && kACol + 32 * sa + 32 <= kTmemCols &&
                                         kDCol + kTileM <= kACol,
                                     P.err, &S.abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (!(ok = wait_or_abort(XPRE ? &S.x_full[sx] : &S.x_conv[sx], (xc / kXStages) & 1, S, P.err)))
                        break;
                    if (!(ok = wait_or_abort(&S.a_full[sa], (ac / kAStages) & 1, S, P.err))) break;
                    tc_fence_after();
                    const uint64_t bdesc = sw128_desc(S.x[sx]);
                    #pragma unroll
                    for (int j = 0; j < 4; ++j)   // K = 16 per MMA: +8 tensor-memory columns, +32 bytes
                        tc_mma_ts(tmem + kDCol, tmem + kACol + 32 * sa + 8 * j, bdesc + 2 * j, kIdesc,
                                  (ks | j) != 0);
                    tc_commit(&S.x_empty[sx]);
                    tc_commit(&S.a_empty[sa]);
                    ++xc;
                    ++ac;
                }
                if (ok) tc_commit(&S.d_full);
            }
            // every MMA issued so far has completed once this commit arrives
            tc_commit(&S.mma_done);
            wait_or_abort(&S.mma_done, 0, S, P.err) || mbar_wait(&S.mma_done, 0, P.err);
        }
    } else if (warp >= kWarpDeq0 && warp < kWarpDeq0 + kNumDeq) {
        const int quad = warp & 3;   // tensor-memory lanes [32*quad, 32*quad + 32)
        const int row = 32 * quad + lane;
        uint32_t rc = 0, ac = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            for (int ks = 0; ks < ksteps && ok; ks += 4) {
                const int s = rc % kRawStages;
                if (Q4_DEBUG_BAD(s < kRawStages && row < kTileN, P.err, &S.abort_flag)) {
                    ok = false;
                    break;
                }
                if (!(ok = wait_or_abort(&S.raw_full[s], (rc / kRawStages) & 1, S, P.err))) break;
                uint32_t raw[36];
                const uint4 *src = reinterpret_cast<const uint4 *>(S.raw[s] + row * kRawRowBytes);
                #pragma unroll
                for (int i = 0; i < 9; ++i) {
                    const uint4 v = src[i];
                    raw[4 * i] = v.x; raw[4 * i + 1] = v.y; raw[4 * i + 2] = v.z; raw[4 * i + 3] = v.w;
                }
                fence_proxy_async_smem();   // the next weight tile may land here
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.raw_empty[s]);
                ++rc;
                #pragma unroll
                for (int sub = 0; sub < 4; ++sub) {      // 64 k = blocks 2*sub, 2*sub+1
                    const int sa = ac % kAStages;
                    if (Q4_DEBUG_BAD(sa < kAStages && kACol + 32 * sa + 32 <= kTmemCols, P.err, &S.abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (!(ok = wait_or_abort(&S.a_empty[sa], ((ac / kAStages) & 1) ^ 1, S, P.err))) break;
                    tc_fence_after();
                    uint32_t cols[32];
                    #pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t dbits, q[4];
                        block_words(raw, 2 * sub + h, dbits, q);
                        const uint32_t d2 = dbits | (dbits << 16);
                        #pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            uint32_t c[4];
                            q4_word_to_fp16(q[w], d2, c);
                            cols[16 * h + 2 * w] = c[0];
                            cols[16 * h + 2 * w + 1] = c[1];
                            cols[16 * h + 8 + 2 * w] = c[2];
                            cols[16 * h + 8 + 2 * w + 1] = c[3];
                        }
                    }
                    tc_st_32(tmem + (uint32_t(32 * quad) << 16) + kACol + 32 * sa, cols);
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.a_full[sa]);
                    ++ac;
                }
            }
        }
    } else if (!XPRE && warp >= kWarpCvt0 && warp < kWarpCvt0 + kNumCvt) {
        // each warp converts rows [32*cw, 32*cw + 32) of the stage; in one pass
        // 8 consecutive lanes take the 8 16-byte chunks of one row (the
        // conversion is chunk-local, so the swizzled order does not matter)
        const int cw = warp - kWarpCvt0;
        uint32_t xc = 0, xbad = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            // the tiles of the first weight-row tile range-check X: every
            // activation row once
            const bool check = t % P.tiles_n == 0;
            for (int ks = 0; ks < ksteps; ++ks) {
                const int s = xc % kXStages;
                if (Q4_DEBUG_BAD(s < kXStages && 32 * cw + 32 <= kTileM, P.err, &S.abort_flag)) {
                    ok = false;
                    break;
                }
                if (!(ok = wait_or_abort(&S.x_full[s], (xc / kXStages) & 1, S, P.err))) break;
                #pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int row = 32 * cw + 4 * it + (lane >> 3);
                    uint4 *p = reinterpret_cast<uint4 *>(S.x[s] + row * 128 + 16 * (lane & 7));
                    const uint4 v = *p;
                    // rows past M are zero-filled by the load
                    if (check) xbad |= x8_fp16_range_bad(v);
                    *p = x8_to_fp16_permuted(v);
                }
                // make the generic-proxy writes visible to the tensor core (async proxy)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.x_conv[s]);
                ++xc;
            }
        }
        if (xbad) atomicOr(P.err, (unsigned)Q4_DEVERR_FP16_RANGE);
    } else {   // epilogue warps
        // lane l of warp quad holds weight row n0 + 32*quad + l of the tile,
        // for the 256 activation rows in 8 chunks of 32 tensor-memory columns
        const int quad = warp & 3;
        const bool swiglu = P.epi == Q4_0_EPI_SWIGLU, residual = P.epi == Q4_0_EPI_RESIDUAL;
        // the residual rows of a tile are asked into L2 while its MMAs run: one
        // 128-byte line (32 weight rows) per activation row and warp
        auto prefetch_r = [&](int t) {
            if (!residual || t >= tiles) return;
            const int n0 = (t % P.tiles_n) * kTileN + 32 * quad, m0 = (t / P.tiles_n) * kTileM;
            if (n0 >= P.N) return;
            for (int m = m0 + lane; m < m0 + kTileM && m < P.M; m += 32)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(P.R + static_cast<int64_t>(m) * P.N + n0));
        };
        prefetch_r(blockIdx.x);
        uint32_t dc = 0, uc = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++dc) {
            if (!wait_or_abort(&S.d_full, dc & 1, S, P.err)) break;
            tc_fence_after();
            const int n0 = (t % P.tiles_n) * kTileN, m0 = (t / P.tiles_n) * kTileM;
            const int n = n0 + 32 * quad + lane;
            if (Q4_DEBUG_BAD(quad < 4 && kDCol + kTileM <= kACol, P.err, &S.abort_flag)) break;
            // a non-finite sum shows in the running value sum_j v[j] * 0
            float nonfinite = 0.f;
            #pragma unroll 1
            for (int c = 0; c < kTileM / 32; ++c) {
                float v[32];
                tc_ld_32(tmem + (uint32_t(32 * quad) << 16) + kDCol + 32 * c, v);
                const int mb = m0 + 32 * c;
                if (n < P.N) {
                    #pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (mb + j < P.M) nonfinite = fmaf(v[j], 0.f, nonfinite);
                }
                if (swiglu) {
                    // rows 0-63 of the tile are the gate rows of features
                    // n0/2 .. n0/2+63 and rows 64-127 their up rows (N % 128 == 0):
                    // warps 0/1 (gate) pair with warps 2/3 (up) on the same 32
                    // features; the gate warp finishes columns 0-15 of the chunk,
                    // the up warp columns 16-31
                    const int xb = uc & 1;
                    const uint32_t xpar = (uc >> 1) & 1;
                    const bool up = quad >= 2;
                    const int fl = 32 * (quad & 1) + lane;
                    if (!(ok = wait_or_abort(&S.xch_empty[xb], xpar ^ 1, S, P.err))) break;
                    // (constant indices into v on both sides: v stays in registers)
                    if (up) {
                        #pragma unroll
                        for (int j = 0; j < 16; ++j) S.xch[xb][j][fl] = v[j];
                    } else {
                        #pragma unroll
                        for (int j = 16; j < 32; ++j) S.xch[xb][j][fl] = v[j];
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.xch_full[xb]);
                    if (!(ok = wait_or_abort(&S.xch_full[xb], xpar, S, P.err))) break;
                    float* const yf = P.Y + (static_cast<int64_t>(mb) * (P.N >> 1) + (n0 >> 1) + fl);
                    const int64_t F = P.N >> 1;
                    if (up) {
                        #pragma unroll
                        for (int j = 16; j < 32; ++j)
                            if (mb + j < P.M) {
                                const float g = S.xch[xb][j][fl];
                                __stcs(yf + j * F, __fdividef(g, 1.0f + __expf(-g)) * v[j]);
                            }
                    } else {
                        #pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (mb + j < P.M) {
                                const float g = v[j];
                                __stcs(yf + j * F, __fdividef(g, 1.0f + __expf(-g)) * S.xch[xb][j][fl]);
                            }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.xch_empty[xb]);
                    ++uc;
                } else if (n < P.N && residual) {
                    // the residual loads of 16 columns before their stores: R may
                    // be Y itself, and loads interleaved with stores to a possible
                    // alias would each wait for the one before
                    #pragma unroll
                    for (int h = 0; h < 32; h += 16) {
                        float r[16];
                        #pragma unroll
                        for (int j = 0; j < 16; ++j)
                            r[j] = mb + h + j < P.M ? __ldcs(P.R + static_cast<int64_t>(mb + h + j) * P.N + n) : 0.f;
                        #pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (mb + h + j < P.M)
                                __stcs(P.Y + static_cast<int64_t>(mb + h + j) * P.N + n, v[h + j] + r[j]);
                    }
                } else if (n < P.N) {
                    #pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (mb + j < P.M)   // streaming store: Y is not read again here, X and W tiles are
                            __stcs(P.Y + static_cast<int64_t>(mb + j) * P.N + n, v[j]);
                }
            }
            if (!ok) break;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.d_empty);
            prefetch_r(t + gridDim.x);
            // a non-finite sum from finite inputs means an fp16 weight
            // overflowed: look at this row's scales (slow path, rare)
            if (nonfinite != 0.f && n < P.N) scan_scales_fp16_range(P.W, n, n + 1, P.N, P.K, P.err);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ---------------------------------------------------------------- host side

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

// bf16 X -> fp16 X' in the permuted k order of the A operand (positions 1 and
// 2 of every 4 swapped), 8 elements per thread.  Exact for |x| in the fp16
// normal range.
// Also flags Q4_DEVERR_FP16_RANGE for values too large for fp16.
__global__ void x_to_fp16_kernel(const uint4 *__restrict__ X, uint4 *__restrict__ Xh, int64_t n8, unsigned *err) {
    uint32_t bad = 0;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 v = __ldg(X + i);
        bad |= x8_fp16_range_bad(v);
        Xh[i] = x8_to_fp16_permuted(v);
    }
    if (bad) atomicOr(err, (unsigned)Q4_DEVERR_FP16_RANGE);
}

}  // namespace

namespace q4 {

bool prefill_supports(const Problem &p) {
    return p.M >= 1 && p.N >= 1 && p.K >= 256 && p.K % 256 == 0 && p.M < (1LL << 31) && p.N < (1LL << 31) &&
           p.K < (1LL << 31) && (reinterpret_cast<uintptr_t>(p.W) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(p.X) & 15) == 0 && tensor_maps_available();
}

// Bytes the fp16 conversion of X writes into a workspace: M*K*2, rounded up
// to 256, whatever M is (a forced tensor-core run of an M <= 32 problem
// converts too).
static int64_t x_conversion_bytes(const Problem &p) { return ((p.M * p.K * 2 + 255) / 256) * 256; }

int64_t prefill_workspace_bytes(const Problem &p) {
    return p.M > 32 ? x_conversion_bytes(p) : 0;
}

int64_t prepared_x_bytes(int64_t M, int64_t K) { return ((M * K * 2 + 255) / 256) * 256; }

cudaError_t launch_prepare_x(const uint16_t *X, int64_t M, int64_t K, void *xh, const DeviceInfo &dev,
                             cudaStream_t s) {
    const int64_t n8 = M * K / 8;
    const int64_t blocks = (n8 + 255) / 256;
    const int grid = static_cast<int>(blocks < dev.sm_count * 8 ? blocks : dev.sm_count * 8);
    if (grid < 1) return cudaSuccess;
    x_to_fp16_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint4 *>(X), static_cast<uint4 *>(xh), n8, dev.err);
    return cudaGetLastError();
}

// The tensor-core kernel on X already in fp16 (xh != nullptr: the pre-pass's
// layout) or on bf16 X converted tile by tile (xh == nullptr).
static cudaError_t launch_prefill_kernel(const Problem &p, const void *xh, const DeviceInfo &dev, cudaStream_t s) {
    const bool xpre = xh != nullptr;
    PrefillParams local;
    std::memset(&local, 0, sizeof(local));
    if (!get_tensor_map(&local.tmap_x, xpre ? xh : p.X, p.M, p.K,
                        xpre ? kMapActivationsF16Sw128 : kMapActivationsSw128) ||
        !get_tensor_map(&local.tmap_w, p.W, p.N, p.K / 32 * 18, kMapWeights128Prefill))
        return cudaErrorInvalidValue;
    local.Y = p.Y;
    local.W = p.W;
    local.R = p.R;
    local.epi = p.epi;
    local.err = dev.err;
    local.M = static_cast<int>(p.M);
    local.N = static_cast<int>(p.N);
    local.K = static_cast<int>(p.K);
    local.tiles_n = static_cast<int>((p.N + kTileN - 1) / kTileN);
    local.tiles_m = static_cast<int>((p.M + kTileM - 1) / kTileM);
    const int tiles = local.tiles_n * local.tiles_m;
    const int grid = tiles < dev.sm_count ? tiles : dev.sm_count;
    if (xpre) {
        static q4::DeviceOnce configured;
        cudaError_t e = configured.run(dev.device, [] {
            return cudaFuncSetAttribute(prefill_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(kSmemBytes));
        });
        if (e != cudaSuccess) return e;
        prefill_kernel<true><<<grid, threads<true>(), kSmemBytes, s>>>(local);
    } else {
        static q4::DeviceOnce configured;
        cudaError_t e = configured.run(dev.device, [] {
            return cudaFuncSetAttribute(prefill_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(kSmemBytes));
        });
        if (e != cudaSuccess) return e;
        prefill_kernel<false><<<grid, threads<false>(), kSmemBytes, s>>>(local);
    }
    return cudaGetLastError();
}

cudaError_t launch_prefill(const Problem &p, const DeviceInfo &dev, cudaStream_t s, void *workspace,
                           int64_t workspace_bytes) {
    // the pre-pass runs only when the workspace holds everything it writes;
    // otherwise the kernel converts each X tile in shared memory
    const bool xpre = workspace != nullptr && workspace_bytes >= x_conversion_bytes(p) &&
                      (reinterpret_cast<uintptr_t>(workspace) & 15) == 0;
    if (xpre) {
        cudaError_t e = launch_prepare_x(p.X, p.M, p.K, workspace, dev, s);
        if (e != cudaSuccess) return e;
    }
    return launch_prefill_kernel(p, xpre ? workspace : nullptr, dev, s);
}

cudaError_t launch_prefill_prepared(const Problem &p, const void *xh, const DeviceInfo &dev, cudaStream_t s) {
    return launch_prefill_kernel(p, xh, dev, s);
}

}  // namespace q4
