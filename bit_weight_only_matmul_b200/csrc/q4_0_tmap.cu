// q4_0_tmap.cu -- TMA tensor maps (host side): encoding through the driver
// entry point, and a small cache so that repeated calls on the same weights
// do not re-encode their maps.
#include <cuda.h>

#include <cstring>
#include <mutex>
#include <unordered_map>

#include "q4_0_internal.cuh"
#include "q4_0_tmap.cuh"

namespace {

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder() {
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    });
    return fn;
}

struct Key {
    const void *ptr;
    int64_t rows, cols;
    int kind;
    bool operator==(const Key &o) const { return ptr == o.ptr && rows == o.rows && cols == o.cols && kind == o.kind; }
};
struct KeyHash {
    size_t operator()(const Key &k) const {
        return std::hash<const void *>()(k.ptr) ^ (std::hash<int64_t>()(k.rows) * 31) ^
               (std::hash<int64_t>()(k.cols) * 131) ^ static_cast<size_t>(k.kind);
    }
};

std::mutex g_mu;
std::unordered_map<Key, CUtensorMap, KeyHash> g_cache;
constexpr size_t kMaxCached = 4096;

bool encode(CUtensorMap *out, const Key &k) {
    EncodeTiled enc = encoder();
    if (!enc) return false;
    const cuuint32_t estr[2] = {1, 1};
    if (k.kind == q4::kMapWeights128 || k.kind == q4::kMapWeights128Prefill || k.kind == q4::kMapWeights16 ||
        k.kind == q4::kMapWeights32) {
        // Q4_0 bytes as uint8 [rows = N, cols = K/32*18], box 144 bytes x 128 (16, 32) rows
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(k.cols), static_cast<cuuint64_t>(k.rows)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(k.cols)};
        const cuuint32_t box_rows = k.kind == q4::kMapWeights16 ? 16 : k.kind == q4::kMapWeights32 ? 32 : 128;
        const cuuint32_t box[2] = {144, box_rows};
        return enc(out, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(k.ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    if (k.kind == q4::kMapActivationsSw128 || k.kind == q4::kMapActivationsF16Sw128 ||
        k.kind == q4::kMapXDecode16 || k.kind == q4::kMapXDecode32) {
        // bf16 or fp16 [rows = M, cols = K], box 64 x (256, 16 or 32), 128-byte swizzle; rows
        // past M read as zero
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(k.cols), static_cast<cuuint64_t>(k.rows)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(k.cols) * 2};
        const cuuint32_t rows = k.kind == q4::kMapXDecode16 ? 16 : k.kind == q4::kMapXDecode32 ? 32 : 256;
        const cuuint32_t box[2] = {64, rows};
        const CUtensorMapDataType t = k.kind == q4::kMapActivationsSw128 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
        return enc(out, t, 2, const_cast<void *>(k.ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    return false;
}

}  // namespace

namespace q4 {

bool tensor_maps_available() { return encoder() != nullptr; }

bool get_tensor_map(CUtensorMap *out, const void *ptr, int64_t rows, int64_t cols, int kind) {
    const Key k{ptr, rows, cols, kind};
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_cache.find(k);
    if (it != g_cache.end()) {
        std::memcpy(out, &it->second, sizeof(CUtensorMap));
        return true;
    }
    CUtensorMap m;
    if (!encode(&m, k)) return false;
    if (g_cache.size() >= kMaxCached) g_cache.clear();
    g_cache.emplace(k, m);
    std::memcpy(out, &m, sizeof(CUtensorMap));
    return true;
}

}  // namespace q4
