// q4_0_internal.cuh -- declarations shared by the library's translation units
// and small sm_100a device helpers (mbarrier waits with a bound, bulk copies).
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/q4_0.h"

namespace q4 {

// One GEMM problem as the kernels see it (same fields as q4_0_problem).
struct Problem {
    const uint8_t *W;
    const uint16_t *X;
    float *Y;
    int64_t M, N, K;
    const float *R = nullptr;   // residual (decode epilogue 1)
    int epi = 0;                // decode epilogue: 0 none, 1 + R, 2 SwiGLU of row-interleaved gate/up
};

// Per-device facts cached by the API layer.
struct DeviceInfo {
    int device;
    int sm_count;
    int cc_major, cc_minor;
    size_t smem_optin;         // max dynamic shared memory per block (opt-in)
    unsigned *err;             // device address of the error word
};

// A set-up step done once per device (device indices are below 64, which the
// API layer checks): one bit per device, set once the step succeeded.  Two
// threads that come first at the same time may both run it; every step
// guarded this way is idempotent.
class DeviceOnce {
  public:
    template <class F>
    cudaError_t run(int device, F &&step) {
        const uint64_t bit = uint64_t{1} << (device & 63);
        if (done_.load(std::memory_order_acquire) & bit) return cudaSuccess;
        const cudaError_t e = step();
        if (e == cudaSuccess) done_.fetch_or(bit, std::memory_order_release);
        return e;
    }

  private:
    std::atomic<uint64_t> done_{0};
};

// A non-negative per-device figure computed once (same rules as DeviceOnce).
class DeviceValue {
  public:
    DeviceValue() {
        for (auto &v : v_) v.store(-1, std::memory_order_relaxed);
    }
    template <class F>
    int get(int device, F &&compute) {
        std::atomic<int> &slot = v_[device & 63];
        int v = slot.load(std::memory_order_acquire);
        if (v >= 0) return v;
        v = compute();
        slot.store(v, std::memory_order_release);
        return v;
    }

  private:
    std::atomic<int> v_[64];
};

// Launchers (host).  Each returns a cudaError_t from the launch.
cudaError_t launch_pack(const uint8_t *codes, const uint16_t *scales, uint8_t *W,
                        int64_t N, int64_t K, cudaStream_t s);
cudaError_t launch_dequant(const uint8_t *W, float *out, int64_t N, int64_t K, cudaStream_t s);
cudaError_t launch_zero(float *Y, int64_t count, cudaStream_t s);
// One CTA whose thread 0 waits, bounded by limit_ns, on a barrier nothing
// arrives on (self-test of the bounded waits).
cudaError_t launch_selftest_wait(const DeviceInfo &dev, unsigned long long limit_ns, cudaStream_t s);
cudaError_t launch_interleave_gate_up(const uint8_t *Wg, const uint8_t *Wu, uint8_t *Wgu, int64_t F, int64_t K,
                                     cudaStream_t s);
cudaError_t launch_gather(const uint8_t *W, const int32_t *ids, float *out, int64_t T, int64_t V, int64_t D,
                          const DeviceInfo &dev, cudaStream_t s);
cudaError_t launch_quantize(const float *X, uint8_t *W, int64_t N, int64_t K, const DeviceInfo &dev,
                            cudaStream_t s);
cudaError_t launch_generic(const Problem *probs, int count, const DeviceInfo &dev, cudaStream_t s);
// Decode kernel on warp-level mma.sync with fp16 weights (M <= 32), the
// default decode path: every problem must satisfy decode_mma_supports().
bool decode_mma_supports(const Problem &p);
cudaError_t launch_decode_mma(const Problem *probs, int count, const DeviceInfo &dev, cudaStream_t s);
// Decode kernel for M <= 8 (warp-level mma.sync, fp16 weights, 512-k ring
// slots): every problem must satisfy decode_m8_supports().
bool decode_m8_supports(const Problem &p);
cudaError_t launch_decode_m8(const Problem *probs, int count, const DeviceInfo &dev, cudaStream_t s);
// Exact-arithmetic decode kernel on warp-level mma.sync (bf16 (q - 8), fp32
// scale per block; M <= 32): every problem must satisfy decode_supports().
bool decode_supports(const Problem &p);
cudaError_t launch_decode(const Problem *probs, int count, const DeviceInfo &dev, cudaStream_t s);
// Decode kernel on tcgen05 with weights in tensor memory (M <= 32): every
// problem must satisfy decode_tmem_supports().
bool decode_tmem_supports(const Problem &p);
cudaError_t launch_decode_tmem(const Problem *probs, int count, const DeviceInfo &dev, cudaStream_t s);
// Read-only stream of a Q4_0 matrix with the decode kernels' TMA boxes (the
// measurement behind q4_0_stream_read).
bool stream_read_supports(int64_t N, int64_t K);
cudaError_t launch_stream_read(const uint8_t *W, int64_t N, int64_t K, uint32_t *checksum, const DeviceInfo &dev,
                               cudaStream_t s);
// Tensor-core kernel: every problem must satisfy prefill_supports().  With a
// workspace of at least prefill_workspace_bytes() X is converted to fp16 once
// by a pre-pass; without one the kernel converts each X tile it loads.
bool prefill_supports(const Problem &p);
int64_t prefill_workspace_bytes(const Problem &p);
// Device address of this device's copy of the library's fixed scratch array
// (Q4_0_STATIC_WS_BYTES, 256-byte aligned); looked up once per device, with
// `dev` current.
cudaError_t static_workspace(int dev, void **out);
cudaError_t launch_prefill(const Problem &p, const DeviceInfo &dev, cudaStream_t s, void *workspace,
                           int64_t workspace_bytes);
// The two phases of the workspace path as separate launches: X (bf16) to the
// fp16 layout the tensor-core kernel reads, and the kernel on it.
int64_t prepared_x_bytes(int64_t M, int64_t K);
cudaError_t launch_prepare_x(const uint16_t *X, int64_t M, int64_t K, void *xh, const DeviceInfo &dev,
                             cudaStream_t s);
cudaError_t launch_prefill_prepared(const Problem &p, const void *xh, const DeviceInfo &dev, cudaStream_t s);

}  // namespace q4

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------
#ifdef __CUDACC__
namespace q4dev {

// A bounded wait gives up after about this many nanoseconds of global time.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// The first ALIGN-aligned byte of a dynamic shared-memory array, reached by
// offsetting the array itself so that the compiler keeps knowing the pointer
// is in shared memory (a round trip through an integer would make every
// access through it a generic one).
template <int ALIGN>
__device__ __forceinline__ uint8_t *align_smem(uint8_t *base) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(base));
    return base + ((ALIGN - (a & (ALIGN - 1))) & (ALIGN - 1));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's generic-proxy shared-memory accesses before later
// async-proxy ones (TMA and bulk copies).  A consumer that read a slot with
// ordinary loads runs it before releasing the slot to the copy engine: the
// mbarrier release alone does not keep the next copy from landing before
// those loads have read the slot.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile(
        "{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile(
        "{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(
            smem_addr(bar)),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that lets the hardware suspend the thread for up to `hint_ns`
// while the phase is incomplete (a waiting warp then issues nothing).
constexpr uint32_t kSuspendHintNs = 1000000;   // 1 ms
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of an mbarrier to complete, for at most
// kWaitLimitNs (or `limit_ns`).  Returns false (and ORs
// Q4_DEVERR_WAIT_TIMEOUT into *err) if the wait ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, unsigned *err,
                                          unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait_suspend(bar, parity)) {
        if (global_ns() - t0 > limit_ns) {
            atomicOr(err, (unsigned)Q4_DEVERR_WAIT_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Index checks of a debug build (compiled with Q4_DEBUG defined): a failed
// check ORs Q4_DEVERR_DEBUG_CHECK into the error word, sets the CTA's abort
// flag so that the other roles stop at their next wait, and yields true, so
// that the caller skips the access and leaves its loop.  Nothing traps.  In
// the product build the check is the constant false and costs nothing.
__device__ __forceinline__ bool debug_bad(bool bad, unsigned *err, int *abort_flag) {
    if (bad) {
        atomicOr(err, (unsigned)Q4_DEVERR_DEBUG_CHECK);
        *reinterpret_cast<volatile int *>(abort_flag) = 1;
    }
    return bad;
}
#ifdef Q4_DEBUG
#define Q4_DEBUG_BAD(ok_cond, err, abort_flag) (::q4dev::debug_bad(!(ok_cond), (err), (abort_flag)))
#else
#define Q4_DEBUG_BAD(ok_cond, err, abort_flag) false
#endif

// 1-D bulk copy global -> shared, completion counted on an mbarrier.
// dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// The same with the destination given as a 32-bit shared-space address.
__device__ __forceinline__ void bulk_g2s_u32(uint32_t dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// (a & b) | c in one instruction.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

}  // namespace q4dev
#endif
