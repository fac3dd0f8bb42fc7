// select.cuh - per-(sequence, KV head) top-K block selection.
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching, Figure 7: the scores pick the K blocks the next step uses;
// "What they did", item 4: a fixed token budget (K = budget / P blocks).
// Ranking: score descending, ties to the lower block id, -0.0 == +0.0.
//
// One CTA per (b, h).  Scores become monotone 32-bit keys in shared memory;
// an MSB-first 8-bit radix select finds the K-th largest key T and how many
// keys equal to T are needed; keys > T are taken, keys == T are taken in
// block-id order (a block-wide scan); the <= K winners are bitonic-sorted by
// (~key, id) and written in rank order.
#pragma once

#include "common.cuh"

namespace oasis {

constexpr int kSelThreads = 512;
constexpr int kSelMaxK = 1024;

// Inclusive block-wide sum over kSelThreads threads; `tmp` holds 32 ints.
__device__ __forceinline__ int block_inclusive_sum(int v, int* tmp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) tmp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < (blockDim.x >> 5) ? tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xFFFFFFFFu, w, o);
            if (lane >= o) w += n;
        }
        tmp[lane] = w;
    }
    __syncthreads();
    const int r = v + (warp > 0 ? tmp[warp - 1] : 0);
    __syncthreads();
    return r;
}

// Scratch of select_unit in shared memory.
struct SelScratch {
    int hist[256];
    int tmp[32];
    int chosen, remaining, gt, pad;
};

// Top-K of one (b, h) with NT threads: keys[0, nv) are the monotone keys of
// the valid blocks (in shared memory, written and synced by the caller);
// cand holds next_pow2(min(K, nv)) entries.  Writes out[0, K) (rank order,
// -1 padded) and, if out_s is not NULL, the scores s[id] of the winners.
template <int NT>
__device__ void select_unit(const uint32_t* keys, int nv, int K, unsigned long long* cand, SelScratch* sc,
                            const float* s, int32_t* out, float* out_s) {
    constexpr int kBpt = NT >= 256 ? 1 : 256 / NT;     // histogram bins per thread
    const int tid = threadIdx.x;
    const int take = min(K, nv);
    int kp = 1;
    while (kp < take) kp <<= 1;
    if (tid == 0) sc->gt = 0;
    __syncthreads();

    uint32_t T = 0;
    int need_eq = 0;
    if (nv > K) {
        uint32_t prefix = 0, mask = 0;
        int remaining = K;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += NT) sc->hist[i] = 0;
            __syncthreads();
            for (int i = tid; i < nv; i += NT) {
                const uint32_t u = keys[i];
                if ((u & mask) == prefix) atomicAdd(&sc->hist[(u >> shift) & 0xFF], 1);
            }
            __syncthreads();
            // suffix sums over bins (bin 255 first): thread t holds bins 255-t*kBpt-k
            int c[kBpt];
            int cnt = 0;
#pragma unroll
            for (int k = 0; k < kBpt; ++k) {
                const int idx = tid * kBpt + k;
                c[k] = idx < 256 ? sc->hist[255 - idx] : 0;
                cnt += c[k];
            }
            const int incl = block_inclusive_sum(cnt, sc->tmp);
            int above = incl - cnt;                     // keys in bins above this thread's first bin
#pragma unroll
            for (int k = 0; k < kBpt; ++k) {
                const int idx = tid * kBpt + k;
                if (idx < 256 && above + c[k] >= remaining && above < remaining) {
                    sc->chosen = 255 - idx;
                    sc->remaining = remaining - above;
                }
                above += c[k];
            }
            __syncthreads();
            prefix |= static_cast<uint32_t>(sc->chosen) << shift;
            mask |= 0xFFu << shift;
            remaining = sc->remaining;
            __syncthreads();
        }
        T = prefix;
        need_eq = remaining;
    }

    // Gather the winners.  Keys > T in any order (sorted below); keys == T in
    // block-id order, the first need_eq of them.
    const int per = (nv + NT - 1) / NT;
    const int i0 = tid * per, i1 = min(nv, i0 + per);
    int eq_local = 0;
    for (int i = i0; i < i1; ++i) {
        const uint32_t u = keys[i];
        const bool win = nv <= K || u > T;
        if (win) {
            const int p = atomicAdd(&sc->gt, 1);
            cand[p] = (static_cast<unsigned long long>(~u) << 32) | static_cast<uint32_t>(i);
        } else if (u == T) {
            ++eq_local;
        }
    }
    const int eq_before = block_inclusive_sum(eq_local, sc->tmp) - eq_local;
    const int n_gt = sc->gt;   // == take - need_eq
    if (nv > K) {
        int e = eq_before;
        for (int i = i0; i < i1 && e < need_eq; ++i) {
            const uint32_t u = keys[i];
            if (u == T) {
                cand[n_gt + e] = (static_cast<unsigned long long>(~u) << 32) | static_cast<uint32_t>(i);
                ++e;
            }
        }
    }
    for (int i = take + tid; i < kp; i += NT) cand[i] = ~0ull;
    __syncthreads();

    // Bitonic sort of kp entries, ascending (~key, id) = score desc, id asc.
    for (int k = 2; k <= kp; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < kp; i += NT) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const unsigned long long x = cand[i], y = cand[ixj];
                    const bool up = (i & k) == 0;
                    if ((x > y) == up) {
                        cand[i] = y;
                        cand[ixj] = x;
                    }
                }
            }
            __syncthreads();
        }
    }

    for (int i = tid; i < K; i += NT) {
        if (i < take) {
            const int id = static_cast<int>(cand[i] & 0xFFFFFFFFu);
            out[i] = id;
            if (out_s) out_s[i] = __ldcg(s + id);
        } else {
            out[i] = -1;
            if (out_s) out_s[i] = -__int_as_float(0x7f800000);
        }
    }
}

__global__ void __launch_bounds__(kSelThreads) select_topk_kernel(Dims d, const float* __restrict__ scores,
                                                                  const int32_t* __restrict__ ctx_len,
                                                                  int32_t* __restrict__ sel,
                                                                  float* __restrict__ sel_score) {
    extern __shared__ uint32_t keys[];                 // [N]
    __shared__ unsigned long long cand[kSelMaxK];
    __shared__ SelScratch sc;
    const int tid = threadIdx.x;
    const int bh = blockIdx.x, b = bh / d.Hkv;
    const int nv = n_valid_blocks(ctx_len[b], d.N);
    const float* s = scores + static_cast<long long>(bh) * d.N;
    for (int i = tid; i < nv; i += kSelThreads) keys[i] = ordered_key(s[i]);
    __syncthreads();
    select_unit<kSelThreads>(keys, nv, d.K, cand, &sc, s, sel + static_cast<long long>(bh) * d.K,
                             sel_score ? sel_score + static_cast<long long>(bh) * d.K : nullptr);
}

}  // namespace oasis
