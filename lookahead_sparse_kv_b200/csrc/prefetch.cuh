// prefetch.cuh - host-to-HBM block gather through mapped pinned memory.
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching, Figure 7 (the chosen blocks come in from the CPU-side KV cache
// ahead of use) and Figure 8 (the copy for step t+1 runs in the background
// once step t has selected).
//
// The kernel reads the pinned host KV directly over PCIe (zero-copy) and
// writes each 8 KiB block into its pool slot, so the gather stays ordered on
// the stream after the planner with no host round trip.  It is persistent
// and small on purpose: 16 CTAs, each thread keeping eight 16-B loads in
// flight (two blocks per CTA at a time), which covers the link's
// bandwidth-delay product (~55 GB/s x a few microseconds).  Measured on B200:
// 16, 32 and 64 CTAs all gather at 51 GB/s, 8 at 45 GB/s; and an attention or
// scoring CTA that shares an SM with a gather CTA runs 1.4-2.5x slower, so
// the fewer SMs the gather occupies the better.  It keeps to 48 registers a
// thread (launch bound of 10 CTAs per SM) and 4 KB of shared memory, so it
// fits beside a scoring CTA.  Only real fetches are visited: a CTA takes the prefix sum of
// the units' fetch counts (1,024 units per pass, in shared memory), numbers
// the fetches of all units consecutively, and takes every gridDim-th pair;
// a binary search over the prefix maps a fetch number back to (unit, entry).
// So the work is even across CTAs however the fetches fall on units, and a
// large cap C costs nothing for the entries it leaves empty.
#pragma once

#include "common.cuh"

namespace oasis {

constexpr int kPrefetchThreads = 128;
constexpr int kPrefetchCtas = 16;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

constexpr int kPrefetchVec = kBlockBytes / 16 / kPrefetchThreads;   // 4 vectors per thread per block
constexpr int kPrefetchChunk = 1024;                                // units per prefix pass
constexpr int kPrefetchPer = kPrefetchChunk / kPrefetchThreads;     // units per thread in the scan

// Unit u of the chunk holding fetch number r (0 <= r < s_pre[nu]): the last
// u with s_pre[u] <= r; units without fetches share their successor's prefix.
__device__ __forceinline__ int prefetch_unit_of(const int* s_pre, int nu, int r) {
    int lo = 0, hi = nu;          // s_pre[lo] <= r < s_pre[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_pre[mid] <= r) lo = mid; else hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(kPrefetchThreads, 10) prefetch_kernel(Dims d, const uint4* __restrict__ host_kv,
                                                                    const int32_t* __restrict__ fetch_slot,
                                                                    const int32_t* __restrict__ fetch_block,
                                                                    const int32_t* __restrict__ n_fetch,
                                                                    uint4* __restrict__ pool) {
    __shared__ int s_pre[kPrefetchChunk + 1];       // exclusive prefix of the chunk's fetch counts
    __shared__ int s_warp[kPrefetchThreads / 32];
    const int units = d.B * d.Hkv;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    long long base = 0;                             // fetches of the units before this chunk
    for (int cu = 0; cu < units; cu += kPrefetchChunk) {
        const int nu = min(kPrefetchChunk, units - cu);
        // block-wide exclusive scan of the clamped counts, kPrefetchPer units per thread
        int loc[kPrefetchPer];
        int run = 0;
#pragma unroll
        for (int k = 0; k < kPrefetchPer; ++k) {
            const int u = t * kPrefetchPer + k;
            loc[k] = run;
            run += u < nu ? min(max(__ldg(n_fetch + cu + u), 0), d.C) : 0;
        }
        int x = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        int before = 0, tot = 0;
#pragma unroll
        for (int w = 0; w < kPrefetchThreads / 32; ++w) {
            before += w < warp ? s_warp[w] : 0;
            tot += s_warp[w];
        }
        const int excl = before + x - run;
#pragma unroll
        for (int k = 0; k < kPrefetchPer; ++k) s_pre[t * kPrefetchPer + k] = excl + loc[k];
        if (t == 0) s_pre[kPrefetchChunk] = tot;
        __syncthreads();
        // fetch pairs q (fetches 2q, 2q+1 in global numbering) with q % gridDim.x == blockIdx.x
        const long long q_lo = base >> 1;
        long long q = q_lo + ((static_cast<long long>(blockIdx.x) - q_lo % gridDim.x + gridDim.x) % gridDim.x);
        for (; 2 * q < base + tot; q += gridDim.x) {
            const uint4 *s0 = nullptr, *s1 = nullptr;
            uint4 *d0 = nullptr, *d1 = nullptr;
            bool v[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const long long r = 2 * q + j - base;
                v[j] = r >= 0 && r < tot;
                if (!v[j]) continue;
                const int u = prefetch_unit_of(s_pre, nu, static_cast<int>(r));
                const int i = static_cast<int>(r) - s_pre[u];
                const long long e = static_cast<long long>(cu + u) * d.C + i;
                const int blk = __ldg(fetch_block + e), slot = __ldg(fetch_slot + e);
                if (blk < 0 || blk >= d.N || slot < 0 || slot >= d.K) {
                    if (t == 0) raise_dev_error(OASIS_DEVERR_ID_RANGE);
                    v[j] = false;
                    continue;
                }
                const uint4* src = host_kv + (static_cast<long long>(cu + u) * d.N + blk) * (kBlockBytes / 16);
                uint4* dst = pool + (static_cast<long long>(cu + u) * d.K + slot) * (kBlockBytes / 16);
                if (j == 0) { s0 = src; d0 = dst; } else { s1 = src; d1 = dst; }
            }
            uint4 a[kPrefetchVec], c[kPrefetchVec];
#pragma unroll
            for (int k = 0; k < kPrefetchVec; ++k) {
                if (v[0]) a[k] = ld_stream(s0 + t + k * kPrefetchThreads);
                if (v[1]) c[k] = ld_stream(s1 + t + k * kPrefetchThreads);
            }
#pragma unroll
            for (int k = 0; k < kPrefetchVec; ++k) {
                if (v[0]) d0[t + k * kPrefetchThreads] = a[k];
                if (v[1]) d1[t + k * kPrefetchThreads] = c[k];
            }
        }
        base += tot;
        __syncthreads();                            // s_pre / s_warp are rewritten by the next pass
    }
}

}  // namespace oasis
