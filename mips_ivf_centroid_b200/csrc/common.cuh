// Device helpers shared by the search kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace ah {

constexpr int kCenters = 16;          // 16 centers per block -> 4-bit codes
constexpr int kTile = 32;             // slots per code tile (one warp)
constexpr int kWarp = 32;

// Device error codes written to the per-index error word (first error wins).
enum DeviceError : int {
    kDevOk = 0,
    kDevCandOverflow = 1,   // candidate buffer still overflowing after the last redo round
    kDevBadLeaf = 2,        // a leaf id outside [0, NL) reached the scan
    kDevSelectSize = 3,     // a selection asked for more items than it holds
    kDevTimeout = 4,        // a bounded wait (tensor-core pipeline barrier) gave up
};

__device__ __forceinline__ void raise_error(int* err, int code) {
    atomicCAS(err, 0, code);
}

// Order-preserving map of a float to uint32 (larger float -> larger key).
// -0.0 is folded to +0.0 first, so equal scores get equal keys.
__device__ __forceinline__ uint32_t float_key(float s) {
    s = s + 0.0f;
    uint32_t b = __float_as_uint(s);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_float(uint32_t k) {
    uint32_t b = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
    return __uint_as_float(b);
}

// 64-bit selection key: (score key, then lower id wins).
__device__ __forceinline__ uint64_t make_key(uint32_t score_key, int32_t id) {
    return (static_cast<uint64_t>(score_key) << 32) | static_cast<uint32_t>(0xFFFFFFFFu - static_cast<uint32_t>(id));
}
__device__ __forceinline__ int32_t key_id(uint64_t key) {
    return static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(key & 0xFFFFFFFFull));
}
__device__ __forceinline__ uint32_t key_score(uint64_t key) {
    return static_cast<uint32_t>(key >> 32);
}

}  // namespace ah
