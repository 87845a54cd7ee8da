// q4_0_prefill.cu -- tensor-core path for M > 32 (placeholder until the
// tcgen05 kernel lands: no problem is routed here).
#include "q4_0_internal.cuh"

namespace q4 {

bool prefill_supports(const Problem &) { return false; }

cudaError_t launch_prefill(const Problem &, const DeviceInfo &, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace q4
