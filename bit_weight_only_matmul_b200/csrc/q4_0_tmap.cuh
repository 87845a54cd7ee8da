// q4_0_tmap.cuh -- host-side TMA tensor maps (see q4_0_tmap.cu).
#pragma once

#include <cuda.h>
#include <cstdint>

namespace q4 {

enum MapKind {
    kMapWeights128 = 1,          // Q4_0 bytes, box 144 bytes (256 k) x 128 rows
    kMapWeights128Prefill = 2,   // same box, cached separately
    kMapActivationsSw128 = 3,    // bf16 X, box 64 x 256, 128-byte swizzle
    kMapActivationsF16Sw128 = 4, // fp16 X, box 64 x 256, 128-byte swizzle
    kMapXDecode16 = 5,           // bf16 X, box 64 x 16, 128-byte swizzle (decode, M <= 16)
    kMapXDecode32 = 6,           // bf16 X, box 64 x 32, 128-byte swizzle (decode, M <= 32)
    kMapWeights16 = 7,           // Q4_0 bytes, box 144 bytes (256 k) x 16 rows
    kMapWeights32 = 8            // Q4_0 bytes, box 144 bytes (256 k) x 32 rows
};

bool tensor_maps_available();
// The map of `ptr` viewed as [rows, cols] (cols in elements of the kind's
// type); cached per (ptr, rows, cols, kind).  False if it cannot be encoded.
bool get_tensor_map(CUtensorMap *out, const void *ptr, int64_t rows, int64_t cols, int kind);

}  // namespace q4
