// summaries.cuh - per-block key min/max summaries (build and append).
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching, Figure 7 (left): the GPU holds keys compressed by per-block
// min/max pooling next to the sparse working set.  The summaries of all N
// blocks stay resident in HBM; decoding folds each appended key row in.
#pragma once

#include "common.cuh"

namespace oasis {

// 16 threads per KV block, each owning 8 channels (one 16-B vector), so a
// group reads each 256-B token row of the block as one coalesced segment.
// The source may be device memory or mapped pinned host memory.
constexpr int kSumThreads = 256;
constexpr int kSumGroups = kSumThreads / 16;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = bf16_lo(w[i]);
        f[2 * i + 1] = bf16_hi(w[i]);
    }
}

// Values are exact bf16, so the top half of the fp32 bit pattern is the bf16.
__device__ __forceinline__ uint4 f32x8_to_bf16(const float (&f)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[i] = (__float_as_uint(f[2 * i]) >> 16) | (__float_as_uint(f[2 * i + 1]) & 0xFFFF0000u);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void __launch_bounds__(kSumThreads) build_summaries_kernel(Dims d, const uint4* __restrict__ kv,
                                                                      const int32_t* __restrict__ ctx_len,
                                                                      int first_block, int n_blocks,
                                                                      uint4* __restrict__ kmin,
                                                                      uint4* __restrict__ kmax) {
    const long long item = static_cast<long long>(blockIdx.x) * kSumGroups + threadIdx.x / 16;
    const int c16 = threadIdx.x & 15;
    const long long total = static_cast<long long>(d.B) * d.Hkv * n_blocks;
    if (item >= total) return;
    const int n = first_block + static_cast<int>(item % n_blocks);
    const long long bh = item / n_blocks;
    const int b = static_cast<int>(bh / d.Hkv);
    const int valid = min(kBlockTokens, ctx_len[b] - n * kBlockTokens);
    if (valid <= 0) return;
    // K rows of block n: 16 rows of 16 uint4.
    const uint4* src = kv + (bh * d.N + n) * (kBlockBytes / 16);
    float mn[8], mx[8];
    bf16x8_to_f32(src[c16], mn);
#pragma unroll
    for (int i = 0; i < 8; ++i) mx[i] = mn[i];
    for (int t = 1; t < valid; ++t) {
        float f[8];
        bf16x8_to_f32(src[t * 16 + c16], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            mn[i] = fminf(mn[i], f[i]);
            mx[i] = fmaxf(mx[i], f[i]);
        }
    }
    const long long o = (bh * d.N + n) * 16 + c16;
    kmin[o] = f32x8_to_bf16(mn);
    kmax[o] = f32x8_to_bf16(mx);
}

// One CTA of 32 threads per (sequence, KV head); threads 0-15 own 8 channels.
__global__ void __launch_bounds__(32) append_kv_kernel(Dims d, const uint4* __restrict__ k_new,
                                                       const uint4* __restrict__ v_new,
                                                       const int32_t* __restrict__ ctx_len,
                                                       int32_t* __restrict__ ctx_len_out, uint4* host_kv,
                                                       uint4* __restrict__ kmin, uint4* __restrict__ kmax,
                                                       const int32_t* __restrict__ slot_table,
                                                       uint4* __restrict__ pool) {
    const int bh = blockIdx.x;
    const int b = bh / d.Hkv;
    const int lane = threadIdx.x;
    const int pos = ctx_len[b];
    const int n = pos / kBlockTokens, t = pos % kBlockTokens;
    if (pos < 0 || n >= d.N) {
        if (lane == 0) raise_dev_error(OASIS_DEVERR_APPEND_FULL);
        return;
    }
    // Which pool slot (if any) holds block n: warp-wide search of the slot table.
    int slot = -1;
    if (pool != nullptr) {
        for (int s0 = 0; s0 < d.K && slot < 0; s0 += 32) {
            const int s = s0 + lane;
            const bool hit = s < d.K && slot_table[static_cast<long long>(bh) * d.K + s] == n;
            const unsigned m = __ballot_sync(0xFFFFFFFFu, hit);
            if (m) slot = s0 + __ffs(m) - 1;
        }
    }
    if (lane < 16) {
        const uint4 kr = k_new[static_cast<long long>(bh) * 16 + lane];
        const uint4 vr = v_new[static_cast<long long>(bh) * 16 + lane];
        if (host_kv != nullptr) {
            uint4* blk = host_kv + (static_cast<long long>(bh) * d.N + n) * (kBlockBytes / 16);
            blk[t * 16 + lane] = kr;
            blk[(kBlockTokens + t) * 16 + lane] = vr;
        }
        const long long o = (static_cast<long long>(bh) * d.N + n) * 16 + lane;
        if (t == 0) {
            kmin[o] = kr;
            kmax[o] = kr;
        } else {
            float a[8], lo[8], hi[8];
            bf16x8_to_f32(kr, a);
            bf16x8_to_f32(kmin[o], lo);
            bf16x8_to_f32(kmax[o], hi);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                lo[i] = fminf(lo[i], a[i]);
                hi[i] = fmaxf(hi[i], a[i]);
            }
            kmin[o] = f32x8_to_bf16(lo);
            kmax[o] = f32x8_to_bf16(hi);
        }
        if (slot >= 0) {
            uint4* dst = pool + (static_cast<long long>(bh) * d.K + slot) * (kBlockBytes / 16);
            dst[t * 16 + lane] = kr;
            dst[(kBlockTokens + t) * 16 + lane] = vr;
        }
    }
    if (ctx_len_out != nullptr && lane == 0 && bh % d.Hkv == 0) ctx_len_out[b] = pos + 1;
}

}  // namespace oasis
