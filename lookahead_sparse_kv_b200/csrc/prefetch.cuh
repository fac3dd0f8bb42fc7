// prefetch.cuh - host-to-HBM block gather through mapped pinned memory.
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching, Figure 7 (selected blocks are prefetched from the CPU cache)
// and Figure 8 (the transfer for step t+1 runs in the background after step
// t's selection).
//
// The kernel reads the pinned host KV directly over PCIe (zero-copy) and
// writes each 8 KiB block into its pool slot, so the gather stays ordered on
// the stream after the planner with no host round trip.  It is persistent
// and small on purpose: a few dozen CTAs walk the (b, h, i) fetch entries two
// at a time, interleaved across the grid, each thread keeping eight 16-B
// loads in flight, which covers the link's bandwidth-delay product
// (~55 GB/s x a few microseconds) while leaving the SMs (and their register
// files) to the attention and scoring kernels that run beside it.  Entries
// past a unit's n_fetch cost a compare against a cached count, so a large
// cap C stays cheap.
#pragma once

#include "common.cuh"

namespace oasis {

constexpr int kPrefetchThreads = 128;
constexpr int kPrefetchCtas = 32;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

constexpr int kPrefetchVec = kBlockBytes / 16 / kPrefetchThreads;   // 4 vectors per thread per block

// Fetch entry v = u*C + i of unit u: source and destination blocks, or false
// if i is past the unit's fetch count (n: n_fetch[u], cached by the caller).
__device__ __forceinline__ bool prefetch_entry(const Dims& d, unsigned v, const uint4* host_kv,
                                               const int32_t* fetch_slot, const int32_t* fetch_block,
                                               const int32_t* n_fetch, int* cached_u, int* cached_n,
                                               const uint4** src, uint4** dst, uint4* pool) {
    const unsigned C = static_cast<unsigned>(d.C);
    const int u = static_cast<int>(v / C), i = static_cast<int>(v - static_cast<unsigned>(u) * C);
    if (u != *cached_u) {
        *cached_u = u;
        *cached_n = min(__ldg(n_fetch + u), d.C);
    }
    if (i >= *cached_n) return false;
    const int blk = __ldg(fetch_block + v), slot = __ldg(fetch_slot + v);
    if (blk < 0 || blk >= d.N || slot < 0 || slot >= d.K) {
        if (threadIdx.x == 0) raise_dev_error(OASIS_DEVERR_ID_RANGE);
        return false;
    }
    *src = host_kv + (static_cast<long long>(u) * d.N + blk) * (kBlockBytes / 16);
    *dst = pool + (static_cast<long long>(u) * d.K + slot) * (kBlockBytes / 16);
    return true;
}

__global__ void __launch_bounds__(kPrefetchThreads) prefetch_kernel(Dims d, const uint4* __restrict__ host_kv,
                                                                    const int32_t* __restrict__ fetch_slot,
                                                                    const int32_t* __restrict__ fetch_block,
                                                                    const int32_t* __restrict__ n_fetch,
                                                                    uint4* __restrict__ pool) {
    // entries < 2^31: B*Hkv <= 65535 and C <= 1024 (host check)
    const unsigned total = static_cast<unsigned>(d.B * d.Hkv) * static_cast<unsigned>(d.C);
    const int t = threadIdx.x;
    int cu0 = -1, cn0 = 0, cu1 = -1, cn1 = 0;
    for (unsigned e0 = 2u * blockIdx.x; e0 < total; e0 += 2u * gridDim.x) {
        const uint4 *s0 = nullptr, *s1 = nullptr;
        uint4 *d0 = nullptr, *d1 = nullptr;
        const bool v0 = prefetch_entry(d, e0, host_kv, fetch_slot, fetch_block, n_fetch, &cu0, &cn0, &s0, &d0, pool);
        const bool v1 = e0 + 1 < total && prefetch_entry(d, e0 + 1, host_kv, fetch_slot, fetch_block, n_fetch,
                                                         &cu1, &cn1, &s1, &d1, pool);
        uint4 a[kPrefetchVec], c[kPrefetchVec];
#pragma unroll
        for (int k = 0; k < kPrefetchVec; ++k) {
            if (v0) a[k] = ld_stream(s0 + t + k * kPrefetchThreads);
            if (v1) c[k] = ld_stream(s1 + t + k * kPrefetchThreads);
        }
#pragma unroll
        for (int k = 0; k < kPrefetchVec; ++k) {
            if (v0) d0[t + k * kPrefetchThreads] = a[k];
            if (v1) d1[t + k * kPrefetchThreads] = c[k];
        }
    }
}

}  // namespace oasis
