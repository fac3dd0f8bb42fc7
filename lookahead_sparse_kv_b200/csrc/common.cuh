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

// Waits unless the CTA has given up; a wait that runs out flags the CTA and
// the device error word.  Returns whether the awaited phase completed.
__device__ __forceinline__ bool cta_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity)) return true;
    *abort_flag = 1;
    raise_dev_error(OASIS_DEVERR_TIMEOUT);
    return false;
}

// A group of NT threads working on one (sequence, KV head) together: the
// whole CTA (CtaGroup), or NT threads starting at thread kFirst that meet at
// named barrier kBar (WarpGroup; the other warps of the CTA go on meanwhile).
template <int NT>
struct CtaGroup {
    static constexpr int kThreads = NT;
    __device__ __forceinline__ static int tid() { return static_cast<int>(threadIdx.x); }
    __device__ __forceinline__ static void sync() { __syncthreads(); }
};

template <int NT, int kBar, int kFirst>
struct WarpGroup {
    static constexpr int kThreads = NT;
    __device__ __forceinline__ static int tid() { return static_cast<int>(threadIdx.x) - kFirst; }
    __device__ __forceinline__ static void sync() { asm volatile("bar.sync %0, %1;" ::"n"(kBar), "n"(NT) : "memory"); }
};

// Exclusive sum of v over the group, in thread order; *total gets the sum of
// all.  tmp: 32 ints of shared memory.  Every thread of the group calls it.
template <class Grp>
__device__ __forceinline__ int group_excl_sum(int v, int* tmp, int* total) {
    constexpr int kWarps = Grp::kThreads / 32;
    const int t = Grp::tid(), lane = t & 31, warp = t >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += n;
    }
    if (lane == 31) tmp[warp] = x;
    Grp::sync();
    if (warp == 0) {
        int w = lane < kWarps ? tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xFFFFFFFFu, w, o);
            if (lane >= o) w += n;
        }
        tmp[lane] = w;
    }
    Grp::sync();
    const int incl = x + (warp > 0 ? tmp[warp - 1] : 0);
    *total = tmp[kWarps - 1];
    Grp::sync();
    return incl - v;
}

}  // namespace oasis
