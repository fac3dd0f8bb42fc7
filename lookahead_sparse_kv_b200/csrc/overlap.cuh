// overlap.cuh - agreement of two block-id lists per (sequence, KV head).
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching, Figure 4 (how well the previous token and a lookahead token
// each predict the top-K blocks) and Figure 6 (overlap between the top-K set
// predicted from the draft query and the one the real next query yields):
// count[b][h] = number of distinct block ids of list b[b][h][*] that also
// occur in list a[b][h][*].  -1 entries are empty.
//
// One CTA per (b, h): list a is marked in a bitmap of N bits in shared
// memory, then every id of list b is tested; a second bitmap makes repeated
// ids of b count once.  Integer only.
#pragma once

#include "common.cuh"

namespace oasis {

constexpr int kOverlapThreads = 256;

__global__ void __launch_bounds__(kOverlapThreads) block_overlap_kernel(Dims d, const int32_t* __restrict__ a,
                                                                         const int32_t* __restrict__ b,
                                                                         int32_t* __restrict__ count) {
    extern __shared__ uint32_t bits[];              // [in_a | counted], ceil(N/32) words each
    __shared__ int warp_sum[kOverlapThreads / 32];
    const int words = (d.N + 31) >> 5;
    uint32_t* in_a = bits;
    uint32_t* counted = bits + words;
    const int tid = threadIdx.x;
    const long long base = static_cast<long long>(blockIdx.x) * d.K;
    for (int i = tid; i < 2 * words; i += kOverlapThreads) bits[i] = 0u;
    __syncthreads();
    for (int i = tid; i < d.K; i += kOverlapThreads) {
        const int id = a[base + i];
        if (id < -1 || id >= d.N) {
            raise_dev_error(OASIS_DEVERR_ID_RANGE);
        } else if (id >= 0) {
            atomicOr(&in_a[id >> 5], 1u << (id & 31));
        }
    }
    __syncthreads();
    int n = 0;
    for (int i = tid; i < d.K; i += kOverlapThreads) {
        const int id = b[base + i];
        if (id < -1 || id >= d.N) {
            raise_dev_error(OASIS_DEVERR_ID_RANGE);
        } else if (id >= 0) {
            const uint32_t bit = 1u << (id & 31);
            if ((in_a[id >> 5] & bit) && !(atomicOr(&counted[id >> 5], bit) & bit)) ++n;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xFFFFFFFFu, n, o);
    if ((tid & 31) == 0) warp_sum[tid >> 5] = n;
    __syncthreads();
    if (tid == 0) {
        int s = 0;
#pragma unroll
        for (int w = 0; w < kOverlapThreads / 32; ++w) s += warp_sum[w];
        count[blockIdx.x] = s;
    }
}

}  // namespace oasis
