// common.cuh - shared definitions of the oasis kernels.
#pragma once

#include <cstdint>

#include "oasis.h"
#include "ptx.cuh"

namespace oasis {

constexpr int kHeadDim = 128;      // D
constexpr int kBlockTokens = 16;   // P
constexpr int kBlockBytes = 2 * kBlockTokens * kHeadDim * 2;   // K + V rows, bf16: 8 KiB
constexpr int kRowBytes = kHeadDim * 2;                        // 256 B

// Plain copy of oasis_dims passed by value to kernels.
struct Dims {
    int B, Hq, Hkv, D, P, N, K, Qn, C;
    __host__ __device__ int G() const { return Hq / Hkv; }
};

// One error word per device (bits OASIS_DEVERR_*).  The library is a single
// translation unit (oasis.cu includes every kernel header), so it is defined
// here.
__device__ unsigned int g_oasis_dev_error = 0u;

__device__ __forceinline__ void raise_dev_error(unsigned int bits) { atomicOr(&g_oasis_dev_error, bits); }

__device__ __forceinline__ int n_valid_blocks(int ctx, int N) {
    int nv = (ctx + kBlockTokens - 1) / kBlockTokens;
    return nv < 0 ? 0 : (nv > N ? N : nv);
}

// fp32 -> uint32 key, monotone in the float order; -0.0 and +0.0 map to the
// same key (they compare equal).
__device__ __forceinline__ uint32_t ordered_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace oasis
