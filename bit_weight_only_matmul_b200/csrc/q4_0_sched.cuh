// q4_0_sched.cuh -- pieces of the persistent decode kernel's work
// distribution: the grouped-problem parameter block, the search of an item's
// problem, and a bounded mbarrier wait that also stops when another role has
// aborted.
//
// An item is 128 weight rows x all of K of one problem.  Problems are sorted
// by K (largest first) on the host, so items with long rows come first, and
// items are dealt to the CTAs in boustrophedon order (round r hands item
// r*G + b to CTA b when r is even and to CTA G-1-b when r is odd), which
// evens out the bytes each CTA streams without any global counter.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "q4_0_internal.cuh"

namespace q4dev {

constexpr int kItemRows = 128;   // weight rows per item
constexpr int kStageK = 256;     // k per stage: 8 Q4_0 blocks
constexpr int kStageRowBytes = 144;

struct GroupProblem {
    const uint8_t *W;
    const uint16_t *X;
    float *Y;
    int M, N, K;
    int stages;        // K / 256
    int item_begin;    // first item index of this problem
    const float *R;    // residual added to Y (epilogue kEpiResidual)
    int epi;           // kEpi*: what the item's end does with its sums
};

// Epilogues of a decode item (values of the C ABI's Q4_0_EPI_*).
constexpr int kEpiNone = 0, kEpiResidual = 1, kEpiSwiGLU = 2;

// CAP problems per launch; the weights' TMA maps live in the kernel parameters.
template <int CAP>
struct alignas(64) GroupParams {
    CUtensorMap wmap[CAP];   // Q4_0 bytes [N, K/32*18], box 144 x 128
    int count;
    int total_items;
    unsigned *err;
    GroupProblem p[CAP];
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

// Bounded wait (kWaitLimitNs) that gives up early once *abort_flag is set, and
// sets it (with Q4_DEVERR_WAIT_TIMEOUT in *err) when it runs out itself.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, int *abort_flag, unsigned *err) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait_suspend(bar, parity)) {
        if (*reinterpret_cast<volatile int *>(abort_flag)) return false;
        if (global_ns() - t0 > kWaitLimitNs) {
            atomicOr(err, (unsigned)Q4_DEVERR_WAIT_TIMEOUT);
            *reinterpret_cast<volatile int *>(abort_flag) = 1;
            return false;
        }
    }
    return true;
}

}  // namespace q4dev
