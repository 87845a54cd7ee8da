// q4_0_static_ws.cu -- the fixed device buffer behind q4_0_gemm_static_ws.
//
// Some callers may not allocate device memory at the moment they multiply:
// a real-time audio thread that must not block inside an allocator, a
// process whose device memory is budgeted once at start-up, or code running
// where no allocator is reachable at all.  For them the library keeps one
// scratch array of Q4_0_STATIC_WS_BYTES in its own device image and hands it
// to the tensor-core path as its workspace (the fp16 copy of X).
//
// The array sits in a file of its own so that, under lazy module loading, a
// process that never calls q4_0_gemm_static_ws never pays for it.  The
// runtime gives every device its own copy; the host learns each copy's device
// address once per device with cudaGetSymbolAddress while that device is
// current.  Nothing in the array has to start at zero: every byte a kernel
// reads from it is written earlier in the same call, on the same stream.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "q4_0_internal.cuh"

static __device__ __align__(256) uint8_t q4_0_static_scratch[Q4_0_STATIC_WS_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
std::atomic<void *> g_addr[kMaxDevices];

}  // namespace

namespace q4 {

cudaError_t static_workspace(int dev, void **out) {
    *out = nullptr;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    void *p = g_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_mu);
        p = g_addr[dev].load(std::memory_order_relaxed);
        if (!p) {
            // The caller has made `dev` current.  A failed look-up is not
            // cached: the next call tries again.
            cudaError_t e = cudaGetSymbolAddress(&p, q4_0_static_scratch);
            if (e != cudaSuccess) {
                (void)cudaGetLastError();   // leave no stale error for later launches
                return e;
            }
            g_addr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return cudaSuccess;
}

}  // namespace q4
