// q4_0_api.cu -- the C ABI (include/q4_0.h): argument checks, per-device
// set-up and the choice of kernel for each problem.
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "q4_0_internal.cuh"

// Device error word (one per device that loads the library): kernels OR
// Q4_DEVERR_* bits into it; q4_0_device_error reads and clears it.
__device__ unsigned q4_0_device_error_word = 0;

namespace {

thread_local int g_last_cuda_error = 0;
std::atomic<int> g_force_path{0};

constexpr int kMaxDevices = 64;
std::once_flag g_dev_once[kMaxDevices];
q4::DeviceInfo g_dev[kMaxDevices];
int g_dev_status[kMaxDevices];

int cuda_fail(cudaError_t e) {
    g_last_cuda_error = static_cast<int>(e);
    return Q4_ERR_CUDA;
}

void init_device(int dev) {
    q4::DeviceInfo &d = g_dev[dev];
    d.device = dev;
    cudaDeviceProp prop;
    cudaError_t e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) { g_dev_status[dev] = cuda_fail(e); return; }
    d.sm_count = prop.multiProcessorCount;
    d.cc_major = prop.major;
    d.cc_minor = prop.minor;
    d.smem_optin = prop.sharedMemPerBlockOptin;
    if (prop.major != 10 || prop.minor != 0) { g_dev_status[dev] = Q4_ERR_UNSUPPORTED_DEVICE; return; }
    // The host-side name of a __device__ variable is not a device address:
    // ask the runtime for this device's address of the error word.
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, q4_0_device_error_word);
    if (e != cudaSuccess) { g_dev_status[dev] = cuda_fail(e); return; }
    d.err = static_cast<unsigned *>(p);
    g_dev_status[dev] = Q4_OK;
}

// Current device's info, set up once per device.
int current_device(const q4::DeviceInfo **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return Q4_ERR_UNSUPPORTED_DEVICE;
    std::call_once(g_dev_once[dev], init_device, dev);
    if (g_dev_status[dev] != Q4_OK) return g_dev_status[dev];
    *out = &g_dev[dev];
    return Q4_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(int64_t N, int64_t K) {
    if (N < 0 || K < 0 || N > Q4_0_MAX_DIM || K > Q4_0_MAX_DIM) return Q4_ERR_INVALID_ARG;
    if (K % 32 != 0) return Q4_ERR_INVALID_ARG;
    return Q4_OK;
}

int check_problem(const q4_0_problem &p) {
    if (p.M < 0 || p.M > Q4_0_MAX_DIM) return Q4_ERR_INVALID_ARG;
    int st = check_dims(p.N, p.K);
    if (st != Q4_OK) return st;
    if (p.M == 0 || p.N == 0) return Q4_OK;
    if (!p.Y) return Q4_ERR_INVALID_ARG;
    if (!aligned16(p.Y)) return Q4_ERR_MISALIGNED;
    if (p.K == 0) return Q4_OK;
    if (!p.W || !p.X) return Q4_ERR_INVALID_ARG;
    if (!aligned16(p.W) || !aligned16(p.X)) return Q4_ERR_MISALIGNED;
    return Q4_OK;
}

enum Path { kAuto = 0, kGeneric = 1, kDecode = 2, kTensor = 3, kDecodeExact = 4, kDecodeTmem = 5, kDecodeM8 = 6 };

// The decode problems of one call: M <= 8 on the 512-k-slot kernel, the rest
// (M <= 32) on the kernel with 1-4 n-tiles of X rows.
cudaError_t launch_decode_split(std::vector<q4::Problem> &dec, std::vector<q4::Problem> &wide,
                                const q4::DeviceInfo &dev, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    if (!dec.empty()) e = q4::launch_decode_m8(dec.data(), static_cast<int>(dec.size()), dev, s);
    if (e == cudaSuccess && !wide.empty())
        e = q4::launch_decode_mma(wide.data(), static_cast<int>(wide.size()), dev, s);
    return e;
}

int run_problems(const q4_0_problem *probs, int count, cudaStream_t s, void *ws = nullptr, int64_t ws_bytes = 0) {
    int st = Q4_OK;
    for (int i = 0; i < count; ++i) {
        st = check_problem(probs[i]);
        if (st != Q4_OK) return st;
    }
    bool any = false;
    for (int i = 0; i < count; ++i) any = any || (probs[i].M > 0 && probs[i].N > 0);
    if (!any) return Q4_OK;
    const q4::DeviceInfo *dev = nullptr;
    st = current_device(&dev);
    if (st != Q4_OK) return st;
    const int force = g_force_path.load(std::memory_order_relaxed);
    // per-thread lists, reused from call to call (no allocation once grown)
    static thread_local std::vector<q4::Problem> dec, dm8, dexact, dtmem, gen, ten;
    dec.clear();
    dm8.clear();
    dexact.clear();
    dtmem.clear();
    gen.clear();
    ten.clear();
    for (int i = 0; i < count; ++i) {
        const q4_0_problem &a = probs[i];
        if (a.M == 0 || a.N == 0) continue;
        if (a.K == 0) {
            cudaError_t e = q4::launch_zero(a.Y, a.M * a.N, s);
            if (e != cudaSuccess) return cuda_fail(e);
            continue;
        }
        q4::Problem p{static_cast<const uint8_t *>(a.W), a.X, a.Y, a.M, a.N, a.K};
        const bool dec_ok = q4::decode_mma_supports(p);
        const bool m8_ok = q4::decode_m8_supports(p);
        const bool exact_ok = q4::decode_supports(p);
        const bool tmem_ok = q4::decode_tmem_supports(p);
        const bool ten_ok = q4::prefill_supports(p);
        if (force == kGeneric) gen.push_back(p);
        else if (force == kDecode && dec_ok) dec.push_back(p);
        else if (force == kDecodeM8 && m8_ok) dm8.push_back(p);
        else if (force == kDecodeExact && exact_ok) dexact.push_back(p);
        else if (force == kDecodeTmem && tmem_ok) dtmem.push_back(p);
        else if (force == kTensor && ten_ok) ten.push_back(p);
        else if (p.M <= 8 && m8_ok) dm8.push_back(p);
        else if (p.M <= 32 && dec_ok) dec.push_back(p);
        else if (p.M > 32 && ten_ok) ten.push_back(p);
        else gen.push_back(p);
    }
    cudaError_t e = launch_decode_split(dm8, dec, *dev, s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (!dexact.empty()) e = q4::launch_decode(dexact.data(), static_cast<int>(dexact.size()), *dev, s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (!dtmem.empty()) e = q4::launch_decode_tmem(dtmem.data(), static_cast<int>(dtmem.size()), *dev, s);
    if (e != cudaSuccess) return cuda_fail(e);
    for (const q4::Problem &p : ten) {
        e = q4::launch_prefill(p, *dev, s, ws, ws_bytes);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    if (!gen.empty()) e = q4::launch_generic(gen.data(), static_cast<int>(gen.size()), *dev, s);
    if (e != cudaSuccess) return cuda_fail(e);
    return Q4_OK;
}

}  // namespace

extern "C" {

const char *q4_0_status_string(int status) {
    switch (status) {
        case Q4_OK: return "Q4_OK";
        case Q4_ERR_INVALID_ARG: return "Q4_ERR_INVALID_ARG: invalid argument (null pointer, bad size, K % 32 != 0)";
        case Q4_ERR_MISALIGNED: return "Q4_ERR_MISALIGNED: a pointer is not 16-byte aligned";
        case Q4_ERR_UNSUPPORTED_DEVICE: return "Q4_ERR_UNSUPPORTED_DEVICE: current device is not sm_100 (CC 10.0)";
        case Q4_ERR_CUDA: return "Q4_ERR_CUDA: a CUDA runtime call failed";
        case Q4_ERR_TOO_LARGE:
            return "Q4_ERR_TOO_LARGE: the problem needs more scratch than the library's fixed buffer "
                   "(Q4_0_STATIC_WS_BYTES) holds";
        default: return "unknown q4_0 status";
    }
}

int q4_0_last_cuda_error(void) { return g_last_cuda_error; }

int64_t q4_0_bytes(int64_t N, int64_t K) {
    if (N < 0 || K < 0 || K % 32 != 0) return -1;
    return N * (K / 32) * 18;
}

int q4_0_pack(const uint8_t *codes, const uint16_t *scales, void *W, int64_t N, int64_t K,
              q4_0_stream_t stream) {
    int st = check_dims(N, K);
    if (st != Q4_OK) return st;
    if (N == 0 || K == 0) return Q4_OK;
    if (!codes || !scales || !W) return Q4_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(W)) return Q4_ERR_MISALIGNED;
    const q4::DeviceInfo *dev = nullptr;
    st = current_device(&dev);
    if (st != Q4_OK) return st;
    cudaError_t e = q4::launch_pack(codes, scales, static_cast<uint8_t *>(W), N, K,
                                    reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

int q4_0_dequant(const void *W, float *out, int64_t N, int64_t K, q4_0_stream_t stream) {
    int st = check_dims(N, K);
    if (st != Q4_OK) return st;
    if (N == 0 || K == 0) return Q4_OK;
    if (!W || !out) return Q4_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(out)) return Q4_ERR_MISALIGNED;
    const q4::DeviceInfo *dev = nullptr;
    st = current_device(&dev);
    if (st != Q4_OK) return st;
    cudaError_t e = q4::launch_dequant(static_cast<const uint8_t *>(W), out, N, K,
                                       reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

int q4_0_gemm(const void *W, const uint16_t *X, float *Y, int64_t M, int64_t N, int64_t K,
              q4_0_stream_t stream) {
    q4_0_problem p{W, X, Y, M, N, K};
    return run_problems(&p, 1, reinterpret_cast<cudaStream_t>(stream));
}

int64_t q4_0_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
    if (M < 0 || N < 0 || K < 0 || K % 32 != 0) return -1;
    q4::Problem p{nullptr, nullptr, nullptr, M, N, K};
    return q4::prefill_workspace_bytes(p);
}

int q4_0_gemm_ws(const void *W, const uint16_t *X, float *Y, int64_t M, int64_t N, int64_t K, void *workspace,
                 int64_t workspace_bytes, q4_0_stream_t stream) {
    if (workspace_bytes < 0 || (workspace_bytes > 0 && !workspace)) return Q4_ERR_INVALID_ARG;
    if (workspace && !aligned16(workspace)) return Q4_ERR_MISALIGNED;
    q4_0_problem p{W, X, Y, M, N, K};
    return run_problems(&p, 1, reinterpret_cast<cudaStream_t>(stream), workspace, workspace_bytes);
}

int64_t q4_0_prepared_x_bytes(int64_t M, int64_t K) {
    if (M < 0 || M > Q4_0_MAX_DIM || K < 0 || K > Q4_0_MAX_DIM || K % 256 != 0) return -1;
    return q4::prepared_x_bytes(M, K);
}

int q4_0_prepare_x(const uint16_t *X, int64_t M, int64_t K, void *xh, int64_t xh_bytes, q4_0_stream_t stream) {
    const int64_t need = q4_0_prepared_x_bytes(M, K);
    if (need < 0 || xh_bytes < 0) return Q4_ERR_INVALID_ARG;
    if (M == 0 || K == 0) return Q4_OK;
    if (!X || !xh || xh_bytes < need) return Q4_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(xh)) return Q4_ERR_MISALIGNED;
    const q4::DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != Q4_OK) return st;
    const cudaError_t e = q4::launch_prepare_x(X, M, K, xh, *dev, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

int q4_0_gemm_prepared(const void *W, const void *xh, float *Y, int64_t M, int64_t N, int64_t K,
                       q4_0_stream_t stream) {
    const q4_0_problem base{W, static_cast<const uint16_t *>(xh), Y, M, N, K};
    int st = check_problem(base);
    if (st != Q4_OK) return st;
    if (M == 0 || N == 0) return Q4_OK;
    if (K < 256 || K % 256 != 0) return Q4_ERR_INVALID_ARG;
    q4::Problem p{static_cast<const uint8_t *>(W), static_cast<const uint16_t *>(xh), Y, M, N, K};
    const q4::DeviceInfo *dev = nullptr;
    st = current_device(&dev);
    if (st != Q4_OK) return st;
    if (!q4::prefill_supports(p)) return Q4_ERR_INVALID_ARG;
    const cudaError_t e = q4::launch_prefill_prepared(p, xh, *dev, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

int q4_0_gemm_static_ws(const void *W, const uint16_t *X, float *Y, int64_t M, int64_t N, int64_t K,
                        q4_0_stream_t stream) {
    const int64_t need = q4_0_gemm_workspace_size(M, N, K);
    if (need < 0 || M > Q4_0_MAX_DIM || N > Q4_0_MAX_DIM || K > Q4_0_MAX_DIM) return Q4_ERR_INVALID_ARG;
    if (need > Q4_0_STATIC_WS_BYTES) return Q4_ERR_TOO_LARGE;
    const q4::DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != Q4_OK) return st;
    void *ws = nullptr;
    const cudaError_t e = q4::static_workspace(dev->device, &ws);
    if (e != cudaSuccess) return cuda_fail(e);
    return q4_0_gemm_ws(W, X, Y, M, N, K, ws, Q4_0_STATIC_WS_BYTES, stream);
}

int q4_0_gather(const void *W, const int32_t *ids, float *out, int64_t T, int64_t V, int64_t D,
                q4_0_stream_t stream) {
    if (T < 0 || T > Q4_0_MAX_DIM || V < 0 || V > Q4_0_MAX_DIM) return Q4_ERR_INVALID_ARG;
    int st = check_dims(V, D);
    if (st != Q4_OK) return st;
    if (T == 0 || D == 0) return Q4_OK;
    if (V == 0 || !W || !ids || !out) return Q4_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(out) || (reinterpret_cast<uintptr_t>(ids) & 3u) != 0) return Q4_ERR_MISALIGNED;
    const q4::DeviceInfo *dev = nullptr;
    st = current_device(&dev);
    if (st != Q4_OK) return st;
    cudaError_t e = q4::launch_gather(static_cast<const uint8_t *>(W), ids, out, T, V, D, *dev,
                                      reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

int q4_0_quantize(const float *X, void *W, int64_t N, int64_t K, q4_0_stream_t stream) {
    int st = check_dims(N, K);
    if (st != Q4_OK) return st;
    if (N == 0 || K == 0) return Q4_OK;
    if (!X || !W) return Q4_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(W)) return Q4_ERR_MISALIGNED;
    const q4::DeviceInfo *dev = nullptr;
    st = current_device(&dev);
    if (st != Q4_OK) return st;
    cudaError_t e = q4::launch_quantize(X, static_cast<uint8_t *>(W), N, K, *dev, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

int q4_0_gemm_grouped_ex(const q4_0_problem_ex *problems, int count, q4_0_stream_t stream) {
    if (count < 0 || count > Q4_0_MAX_GROUP || (count > 0 && !problems)) return Q4_ERR_INVALID_ARG;
    if (count == 0) return Q4_OK;
    static thread_local std::vector<q4::Problem> dec, dm8, big;
    dec.clear();
    dm8.clear();
    big.clear();
    for (int i = 0; i < count; ++i) {
        const q4_0_problem_ex &a = problems[i];
        const q4_0_problem base{a.W, a.X, a.Y, a.M, a.N, a.K};
        int st = check_problem(base);
        if (st != Q4_OK) return st;
        if (a.M < 1 || a.N < 1 || a.K < 256 || a.K % 256 != 0) return Q4_ERR_INVALID_ARG;
        if (a.epilogue == Q4_0_EPI_RESIDUAL) {
            if (!a.R) return Q4_ERR_INVALID_ARG;
            if (!aligned16(a.R)) return Q4_ERR_MISALIGNED;
        } else if (a.epilogue == Q4_0_EPI_SWIGLU) {
            if (a.N % 128 != 0) return Q4_ERR_INVALID_ARG;
        } else if (a.epilogue != Q4_0_EPI_NONE) {
            return Q4_ERR_INVALID_ARG;
        }
        q4::Problem p{static_cast<const uint8_t *>(a.W), a.X, a.Y, a.M, a.N, a.K};
        p.R = a.epilogue == Q4_0_EPI_RESIDUAL ? a.R : nullptr;
        p.epi = a.epilogue;
        if (p.M > 32) {   // the tensor-core kernel, its epilogue warps applying the epilogue
            if (!q4::prefill_supports(p)) return Q4_ERR_INVALID_ARG;
            big.push_back(p);
            continue;
        }
        if (!q4::decode_mma_supports(p)) return Q4_ERR_INVALID_ARG;
        const int force = g_force_path.load(std::memory_order_relaxed);
        if (p.M <= 8 && force != kDecode && q4::decode_m8_supports(p)) dm8.push_back(p);
        else dec.push_back(p);
    }
    const q4::DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != Q4_OK) return st;
    cudaError_t e = launch_decode_split(dm8, dec, *dev, reinterpret_cast<cudaStream_t>(stream));
    for (size_t i = 0; i < big.size() && e == cudaSuccess; ++i)
        e = q4::launch_prefill(big[i], *dev, reinterpret_cast<cudaStream_t>(stream), nullptr, 0);
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

int q4_0_interleave_gate_up(const void *W_gate, const void *W_up, void *W_gu, int64_t F, int64_t K,
                            q4_0_stream_t stream) {
    int st = check_dims(2 * F, K);
    if (st != Q4_OK || F < 0 || F % 64 != 0 || K % 256 != 0) return Q4_ERR_INVALID_ARG;
    if (F == 0 || K == 0) return Q4_OK;
    if (!W_gate || !W_up || !W_gu) return Q4_ERR_INVALID_ARG;
    if (!aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_gu)) return Q4_ERR_MISALIGNED;
    const q4::DeviceInfo *dev = nullptr;
    st = current_device(&dev);
    if (st != Q4_OK) return st;
    const cudaError_t e = q4::launch_interleave_gate_up(static_cast<const uint8_t *>(W_gate),
                                                         static_cast<const uint8_t *>(W_up), static_cast<uint8_t *>(W_gu),
                                                         F, K, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

int q4_0_stream_read(const void *W, int64_t N, int64_t K, uint32_t *checksum, q4_0_stream_t stream) {
    int st = check_dims(N, K);
    if (st != Q4_OK) return st;
    if (N == 0 || K == 0) return Q4_OK;
    if (!W || !checksum || K % 256 != 0) return Q4_ERR_INVALID_ARG;
    if (!aligned16(W)) return Q4_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(checksum) & 3u) != 0) return Q4_ERR_MISALIGNED;
    const q4::DeviceInfo *dev = nullptr;
    st = current_device(&dev);
    if (st != Q4_OK) return st;
    if (!q4::stream_read_supports(N, K)) return Q4_ERR_INVALID_ARG;
    const cudaError_t e = q4::launch_stream_read(static_cast<const uint8_t *>(W), N, K, checksum, *dev,
                                                 reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

int q4_0_selftest_wait_timeout(uint32_t limit_us, q4_0_stream_t stream) {
    if (limit_us < 1 || limit_us > 1000000) return Q4_ERR_INVALID_ARG;
    const q4::DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != Q4_OK) return st;
    const cudaError_t e = q4::launch_selftest_wait(*dev, static_cast<unsigned long long>(limit_us) * 1000ull,
                                                   reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? Q4_OK : cuda_fail(e);
}

int q4_0_gemm_grouped(const q4_0_problem *problems, int count, q4_0_stream_t stream) {
    if (count < 0 || count > Q4_0_MAX_GROUP) return Q4_ERR_INVALID_ARG;
    if (count == 0) return Q4_OK;
    if (!problems) return Q4_ERR_INVALID_ARG;
    return run_problems(problems, count, reinterpret_cast<cudaStream_t>(stream));
}

int q4_0_device_error(uint32_t *flags, int clear) {
    if (!flags) return Q4_ERR_INVALID_ARG;
    const q4::DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != Q4_OK) return st;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned v = 0;
    e = cudaMemcpy(&v, dev->err, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e);
    *flags = v;
    if (clear) {
        e = cudaMemset(dev->err, 0, sizeof(unsigned));
        if (e != cudaSuccess) return cuda_fail(e);
        e = cudaDeviceSynchronize();
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return Q4_OK;
}

int q4_0_force_path(int path) {
    if (path < 0 || path > 6) return Q4_ERR_INVALID_ARG;
    g_force_path.store(path, std::memory_order_relaxed);
    return Q4_OK;
}

}  // extern "C"
