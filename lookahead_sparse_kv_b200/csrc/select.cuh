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

// Scratch of select_unit in shared memory.
struct SelScratch {
    int hist[256];
    int tmp[32];
    int chosen, remaining, gt, pad;
};

// Monotone keys of a unit's scores: from shared memory, or computed from the
// fp32 scores in global memory (read through L2) when they do not fit there.
struct SmemKeys {
    const uint32_t* k;
    __device__ __forceinline__ uint32_t operator()(int i) const { return k[i]; }
};
struct GlobalKeys {
    const float* s;
    __device__ __forceinline__ uint32_t operator()(int i) const { return ordered_key(__ldcg(s + i)); }
};

// Top-K of one (b, h) by a group of threads: key(i), i < nv, is the monotone
// key of valid block i (keys in shared memory written and synced by the
// caller); cand holds next_pow2(min(K, nv)) entries.  Writes out[0, K)
// (rank order, -1 padded) and, if out_s is not NULL, the scores s[id] of the
// winners.
template <class Grp, class Key>
__device__ void select_unit(Key key, int nv, int K, unsigned long long* cand, SelScratch* sc, const float* s,
                            int32_t* out, float* out_s) {
    constexpr int NT = Grp::kThreads;
    constexpr int kBpt = NT >= 256 ? 1 : 256 / NT;     // histogram bins per thread
    const int tid = Grp::tid();
    const int take = min(K, nv);
    int kp = 1;
    while (kp < take) kp <<= 1;
    Grp::sync();

    uint32_t T = 0;
    int need_eq = 0;
    if (nv > K && NT <= 128 && nv <= 32 * NT) {
        // small groups: the K-th largest key by bisection on the key value (each
        // thread holds its, at most 32, keys in registers; one barrier per step;
        // padding keys are 0, below every score's key); large groups take the radix
        // passes below
        const int per = (nv + NT - 1) / NT;
        const int i0 = tid * per;
        uint32_t kk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) kk[j] = (j < per && i0 + j < nv) ? key(i0 + j) : 0u;
        uint32_t lo = 0u, hi = 0xFFFFFFFFu;          // count(>= lo) >= K > count(>= hi + 1)
        for (int it = 0; lo < hi; ++it) {
            const uint32_t mid = lo + ((hi - lo) >> 1) + 1u;
            int c = 0;
#pragma unroll
            for (int j = 0; j < 32; ++j) c += kk[j] >= mid ? 1 : 0;
            c = __reduce_add_sync(0xFFFFFFFFu, c);
            if ((tid & 31) == 0) sc->hist[(it & 1) * 32 + (tid >> 5)] = c;
            Grp::sync();
            int tot = 0;
#pragma unroll
            for (int w = 0; w < NT / 32; ++w) tot += sc->hist[(it & 1) * 32 + w];
            if (tot >= K) lo = mid; else hi = mid - 1u;
        }
        T = lo;
        int c = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) c += kk[j] > T ? 1 : 0;
        int gt_all;
        group_excl_sum<Grp>(c, sc->tmp, &gt_all);
        need_eq = K - gt_all;
    } else if (nv > K) {
        uint32_t prefix = 0, mask = 0;
        int remaining = K;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += NT) sc->hist[i] = 0;
            Grp::sync();
            // scores of one unit cluster in a few bins: lanes of a warp that share a
            // bin add to it once (one shared-memory atomic per distinct bin per warp);
            // four keys per thread are read before any is binned
            for (int base = 0; base < nv; base += 4 * NT) {
                uint32_t uk[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = base + k * NT + tid;
                    uk[k] = i < nv ? key(i) : 0u;
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = base + k * NT + tid;
                    const int bin = (i < nv && (uk[k] & mask) == prefix) ? static_cast<int>((uk[k] >> shift) & 0xFF) : -1;
                    const unsigned same = __match_any_sync(0xFFFFFFFFu, bin);
                    if (bin >= 0 && __ffs(same) - 1 == (tid & 31)) atomicAdd(&sc->hist[bin], __popc(same));
                }
            }
            Grp::sync();
            // suffix sums over bins (bin 255 first): thread t holds bins 255-t*kBpt-k
            int c[kBpt];
            int cnt = 0;
#pragma unroll
            for (int k = 0; k < kBpt; ++k) {
                const int idx = tid * kBpt + k;
                c[k] = idx < 256 ? sc->hist[255 - idx] : 0;
                cnt += c[k];
            }
            int total;
            int above = group_excl_sum<Grp>(cnt, sc->tmp, &total);   // keys in bins above this thread's first bin
#pragma unroll
            for (int k = 0; k < kBpt; ++k) {
                const int idx = tid * kBpt + k;
                if (idx < 256 && above + c[k] >= remaining && above < remaining) {
                    sc->chosen = 255 - idx;
                    sc->remaining = remaining - above;
                }
                above += c[k];
            }
            Grp::sync();
            prefix |= static_cast<uint32_t>(sc->chosen) << shift;
            mask |= 0xFFu << shift;
            remaining = sc->remaining;
            Grp::sync();
        }
        T = prefix;
        need_eq = remaining;
    }

    // Gather the winners.  Keys > T in any order (sorted below); keys == T in
    // block-id order, the first need_eq of them.  Each thread takes a
    // contiguous chunk; block scans place the chunks' winners.
    const int per = (nv + NT - 1) / NT;
    const int i0 = tid * per, i1 = min(nv, i0 + per);
    int gt_local = 0, eq_local = 0;
    for (int i = i0; i < i1; ++i) {
        const uint32_t u = key(i);
        if (nv <= K || u > T) ++gt_local;
        else if (u == T) ++eq_local;
    }
    int total;
    int p = group_excl_sum<Grp>(gt_local, sc->tmp, &total);
    if (tid == 0) sc->gt = total;
    for (int i = i0; i < i1 && gt_local > 0; ++i) {
        const uint32_t u = key(i);
        if (nv <= K || u > T) {
            cand[p++] = (static_cast<unsigned long long>(~u) << 32) | static_cast<uint32_t>(i);
            --gt_local;
        }
    }
    const int eq_before = group_excl_sum<Grp>(eq_local, sc->tmp, &total);   // (syncs: sc->gt visible)
    const int n_gt = sc->gt;   // == take - need_eq
    if (nv > K) {
        int e = eq_before;
        for (int i = i0; i < i1 && e < need_eq; ++i) {
            const uint32_t u = key(i);
            if (u == T) {
                cand[n_gt + e] = (static_cast<unsigned long long>(~u) << 32) | static_cast<uint32_t>(i);
                ++e;
            }
        }
    }
    for (int i = take + tid; i < kp; i += NT) cand[i] = ~0ull;
    Grp::sync();

    // Rank order (~key, id) ascending = score desc, id asc.  Up to two winners
    // a thread: each winner's rank is the number of smaller entries (they are
    // distinct); more: bitonic sort of kp entries.
    if (take <= 2 * NT) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int i = tid + h * NT;
            if (i >= take) continue;
            const unsigned long long c = cand[i];
            int rank = 0;
            int j = 0;
#pragma unroll 4
            for (; j + 1 < take; j += 2) {
                const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(cand + j);
                rank += (x.x < c) + (x.y < c);
            }
            if (j < take) rank += cand[j] < c;
            const int id = static_cast<int>(c & 0xFFFFFFFFu);
            out[rank] = id;
            if (out_s) out_s[rank] = __ldcg(s + id);
        }
        for (int i = take + tid; i < K; i += NT) {
            out[i] = -1;
            if (out_s) out_s[i] = -__int_as_float(0x7f800000);
        }
        return;
    }
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
            Grp::sync();
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
    __shared__ __align__(16) unsigned long long cand[kSelMaxK];
    __shared__ SelScratch sc;
    const int tid = threadIdx.x;
    const int bh = blockIdx.x, b = bh / d.Hkv;
    const int nv = n_valid_blocks(ctx_len[b], d.N);
    const float* s = scores + static_cast<long long>(bh) * d.N;
    for (int i = tid; i < nv; i += kSelThreads) keys[i] = ordered_key(s[i]);
    __syncthreads();
    select_unit<CtaGroup<kSelThreads>>(SmemKeys{keys}, nv, d.K, cand, &sc, s, sel + static_cast<long long>(bh) * d.K,
                                       sel_score ? sel_score + static_cast<long long>(bh) * d.K : nullptr);
}

}  // namespace oasis
