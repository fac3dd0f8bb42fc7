// select.cuh - per-(sequence, KV head) top-K block selection.
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching, Figure 7: the scores pick the K blocks the next step uses;
// "What they did", item 4: a fixed token budget (K = budget / P blocks).
// Ranking: score descending, ties to the lower block id, -0.0 == +0.0.
//
// Scores become monotone 32-bit keys.  The group finds the K-th largest key
// T; keys > T are taken, then keys == T in block-id order until K are taken;
// the <= K winners are put in rank order (~key, id) and written out.
//   - Register path (select_unit_regs, up to 64 keys a thread): each thread
//     holds its keys in registers; T comes from a 4-way search on the key
//     value (three pivots a round, one barrier a round, stopping early once a
//     pivot has exactly K keys at or above it).
//   - Shared-memory path (select_unit, any count): an MSB-first 8-bit radix
//     select over keys in shared memory (or read through L2).
#pragma once

#include "common.cuh"

namespace oasis {

constexpr int kSelThreads = 512;
constexpr int kSelMaxK = 1024;

// Scratch of select_unit / select_unit_regs in shared memory.
struct alignas(16) SelScratch {
    int hist[256];
    int cnt[2][16][8];          // register path: per-warp pivot counts, two rounds in flight
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

// Score of a winner from its candidate entry (~key << 32 | id): the key read
// backwards; a zero key is read from the scores, which keep the sign of zero.
__device__ __forceinline__ float cand_score(unsigned long long c, const float* s) {
    const uint32_t k = ~static_cast<uint32_t>(c >> 32);
    if (k == 0x80000000u) return __ldcg(s + static_cast<uint32_t>(c));
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// The take <= K winners in cand[0, take) (any order; cand[take, kp) = ~0,
// written and synced by the caller) go out in rank order: (~key, id)
// ascending = score descending, id ascending.  out[take, K) = -1.  s_out (may
// be NULL): a copy of out in shared memory, synced on return.
template <class Grp>
__device__ void select_finish(unsigned long long* cand, int take, int kp, int K, const float* s, int32_t* out,
                              float* out_s, int32_t* s_out) {
    constexpr int NT = Grp::kThreads;
    const int tid = Grp::tid();
    // Up to two winners a thread: each winner's rank is the number of smaller
    // entries (they are distinct); more: bitonic sort of kp entries.
    if (take <= 2 * NT) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int i = tid + h * NT;
            if (i >= take) continue;
            const unsigned long long c = cand[i];
            int r0 = 0, r1 = 0;
            int j = 0;
#pragma unroll 4
            for (; j + 3 < take; j += 4) {
                const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(cand + j);
                const ulonglong2 y = *reinterpret_cast<const ulonglong2*>(cand + j + 2);
                r0 += (x.x < c) + (x.y < c);
                r1 += (y.x < c) + (y.y < c);
            }
            for (; j < take; ++j) r0 += cand[j] < c;
            const int rank = r0 + r1;
            const int id = static_cast<int>(c & 0xFFFFFFFFu);
            out[rank] = id;
            if (s_out) s_out[rank] = id;
            if (out_s) out_s[rank] = cand_score(c, s);
        }
    } else {
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
        for (int i = tid; i < take; i += NT) {
            const unsigned long long c = cand[i];
            const int id = static_cast<int>(c & 0xFFFFFFFFu);
            out[i] = id;
            if (s_out) s_out[i] = id;
            if (out_s) out_s[i] = cand_score(c, s);
        }
    }
    for (int i = take + tid; i < K; i += NT) {
        out[i] = -1;
        if (s_out) s_out[i] = -1;
        if (out_s) out_s[i] = -__int_as_float(0x7f800000);
    }
    if (s_out) Grp::sync();
}

// Top-K of one (b, h) by a group of threads: key(i), i < nv, is the monotone
// key of valid block i (keys in shared memory written and synced by the
// caller); cand holds next_pow2(min(K, nv)) entries.  Writes out[0, K)
// (rank order, -1 padded), the winners' scores to out_s and a copy of out to
// s_out, either when not NULL (as select_finish).
template <class Grp, class Key>
__device__ void select_unit(Key key, int nv, int K, unsigned long long* cand, SelScratch* sc, const float* s,
                            int32_t* out, float* out_s, int32_t* s_out = nullptr) {
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

    select_finish<Grp>(cand, take, kp, K, s, out, out_s, s_out);
}

// ---------------------------------------------------------------------------
// Register path.  Thread t of the group holds PER keys; its key j is that of
// block rk_block(t, j) = (j / 4) * 4 * NT + 4 * t + j % 4, so the unit is
// read in PER / 4 coalesced passes of 16-B loads.  Blocks >= nv hold key 0
// and real blocks at least 1 (rk_key), so the key alone tells them apart.
template <int NT>
__device__ __forceinline__ int rk_block(int t, int j) { return (j >> 2) * (4 * NT) + 4 * t + (j & 3); }

// ordered_key, with the one float that maps to 0 (the NaN 0xFFFFFFFF) moved
// up to 1 beside its neighbouring NaN
__device__ __forceinline__ uint32_t rk_key(uint32_t k) { return k > 1u ? k : 1u; }

// Keys from fp32 scores s[0, nv) read through L2.  vec4: s is 16-B aligned
// and its row holds a multiple of 4 floats, so a 16-B read that starts below
// nv stays inside the row.
template <class Grp, int PER>
__device__ __forceinline__ void rk_load_scores(uint32_t (&kk)[PER], const float* s, int nv, bool vec4) {
    constexpr int NT = Grp::kThreads;
    const int t = Grp::tid();
    if (vec4) {
        // the raw bits first (every load in flight), then the keys in place
#pragma unroll
        for (int r = 0; r < PER / 4; ++r) {
            const int i = r * 4 * NT + 4 * t;
            const uint4 v = i < nv ? __ldcg(reinterpret_cast<const uint4*>(s + i)) : make_uint4(0u, 0u, 0u, 0u);
            kk[4 * r + 0] = v.x;
            kk[4 * r + 1] = v.y;
            kk[4 * r + 2] = v.z;
            kk[4 * r + 3] = v.w;
        }
#pragma unroll
        for (int j = 0; j < PER; ++j)
            kk[j] = rk_block<NT>(t, j) < nv ? rk_key(ordered_key(__uint_as_float(kk[j]))) : 0u;
    } else {
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int i = rk_block<NT>(t, j);
            kk[j] = i < nv ? rk_key(ordered_key(__ldcg(s + i))) : 0u;
        }
    }
}

// Keys from shared memory (ordered_key values, 16-B aligned, readable up to
// nv rounded up to 4).
template <class Grp, int PER>
__device__ __forceinline__ void rk_load_keys(uint32_t (&kk)[PER], const uint32_t* keys, int nv) {
    constexpr int NT = Grp::kThreads;
    const int t = Grp::tid();
#pragma unroll
    for (int r = 0; r < PER / 4; ++r) {
        const int i = r * 4 * NT + 4 * t;
        const uint4 v = i < nv ? *reinterpret_cast<const uint4*>(keys + i) : make_uint4(0u, 0u, 0u, 0u);
        kk[4 * r + 0] = i + 0 < nv ? rk_key(v.x) : 0u;
        kk[4 * r + 1] = i + 1 < nv ? rk_key(v.y) : 0u;
        kk[4 * r + 2] = i + 2 < nv ? rk_key(v.z) : 0u;
        kk[4 * r + 3] = i + 3 < nv ? rk_key(v.w) : 0u;
    }
}

// Top-K of one (b, h) from register-resident keys (nv <= PER * NT).  cand
// holds next_pow2(min(K, nv)) entries; out, out_s, s_out as in select_finish.
template <class Grp, int PER>
__device__ void select_unit_regs(const uint32_t (&kk)[PER], int nv, int K, unsigned long long* cand, SelScratch* sc,
                                 const float* s, int32_t* out, float* out_s, int32_t* s_out) {
    constexpr int NT = Grp::kThreads, NW = NT / 32;
    static_assert(PER % 4 == 0 && NW <= 16, "register select layout");
    const int tid = Grp::tid(), lane = tid & 31, warp = tid >> 5;
    const int take = min(K, nv);
    int kp = 1;
    while (kp < take) kp <<= 1;

    // T: keys > T are taken, then need_eq keys == T in block order
    uint32_t T = 0;
    if (nv > K) {
        // the bracket [lo, hi]: count(>= lo) >= K > count(>= hi + 1); every pivot
        // is above lo >= 1, so the padding keys (0) are never counted
        uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            mn = min(mn, kk[j] != 0u ? kk[j] : 0xFFFFFFFFu);
            mx = max(mx, kk[j]);
        }
        mn = __reduce_min_sync(0xFFFFFFFFu, mn);
        mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        if (lane == 0) {
            sc->hist[warp] = static_cast<int>(mn);
            sc->hist[32 + warp] = static_cast<int>(mx);
        }
        Grp::sync();
        uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            lo = min(lo, static_cast<uint32_t>(sc->hist[w]));
            hi = max(hi, static_cast<uint32_t>(sc->hist[32 + w]));
        }
        // each round counts the keys at or above NP = 3 pivots spread evenly
        // over (lo, hi] and keeps the quarter that holds the K-th key; a pivot
        // with exactly K keys at or above it ends the search (every key >= it
        // is taken).  (Seven pivots a round took fewer rounds but longer ones:
        // 2.4 against 1.8 us for 2,048 keys on 128 threads.)
        constexpr int NP = 3;
        for (int it = 0;; ++it) {
            if (lo >= hi) {
                T = lo;
                break;
            }
            const unsigned long long span = hi - lo;
            uint32_t pv[NP];
            int c[NP];
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                pv[k] = lo + static_cast<uint32_t>(((k + 1) * span + NP) / (NP + 1));   // in (lo, hi], non-decreasing
                c[k] = 0;
            }
#pragma unroll
            for (int j = 0; j < PER; ++j)
#pragma unroll
                for (int k = 0; k < NP; ++k) c[k] += kk[j] >= pv[k] ? 1 : 0;
#pragma unroll
            for (int k = 0; k < NP; ++k) c[k] = __reduce_add_sync(0xFFFFFFFFu, c[k]);
            int* buf = &sc->cnt[it & 1][warp][0];
            if (lane == 0) {
                *reinterpret_cast<int4*>(buf) = make_int4(c[0], c[1], c[2], NP > 3 ? c[NP > 3 ? 3 : 0] : 0);
                if constexpr (NP > 4)
                    *reinterpret_cast<int4*>(buf + 4) = make_int4(c[NP > 4 ? 4 : 0], c[NP > 5 ? 5 : 0], c[NP > 6 ? 6 : 0], 0);
            }
            Grp::sync();
            int C[NP];
#pragma unroll
            for (int k = 0; k < NP; ++k) C[k] = 0;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const int4 x = *reinterpret_cast<const int4*>(&sc->cnt[it & 1][w][0]);
                C[0] += x.x;
                C[1] += x.y;
                C[2] += x.z;
                if constexpr (NP > 3) C[NP > 3 ? 3 : 0] += x.w;
                if constexpr (NP > 4) {
                    const int4 y = *reinterpret_cast<const int4*>(&sc->cnt[it & 1][w][4]);
                    C[NP > 4 ? 4 : 0] += y.x;
                    C[NP > 5 ? 5 : 0] += y.y;
                    C[NP > 6 ? 6 : 0] += y.z;
                }
            }
            // the largest k with C[k] >= K (C is non-increasing; count(>= lo) >= K)
            int kb = -1;
#pragma unroll
            for (int k = 0; k < NP; ++k) kb = C[k] >= K ? k : kb;
            bool exact = false;
            uint32_t nlo = lo, nhi = hi;
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                if (k == kb) {
                    exact = C[k] == K;
                    nlo = pv[k];
                }
                if (k == kb + 1) nhi = pv[k] - 1u;
            }
            if (exact) {
                T = nlo - 1u;
                break;
            }
            lo = nlo;
            hi = nhi;
        }
    }

    // gather: keys > T anywhere in cand[0, n_gt); keys == T after them (with
    // nv <= K every real key is taken: T = 0 and no key equals it)
    int gt = 0, eq = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        gt += kk[j] > T ? 1 : 0;
        eq += (T != 0u && kk[j] == T) ? 1 : 0;
    }
    int tot;
    // both counts in one scan: each total is at most nv <= 32768 < 2^16
    const uint32_t ex = static_cast<uint32_t>(group_excl_sum<Grp>(gt | (eq << 16), sc->tmp, &tot));
    const int n_gt = static_cast<int>(static_cast<uint32_t>(tot) & 0xFFFFu);
    const int n_eq = static_cast<int>(static_cast<uint32_t>(tot) >> 16);
    const int need_eq = nv > K ? K - n_gt : 0;
    int pg = static_cast<int>(ex & 0xFFFFu);
#pragma unroll
    for (int j = 0; j < PER; ++j)
        if (kk[j] > T)
            cand[pg++] = (static_cast<unsigned long long>(~kk[j]) << 32) | static_cast<uint32_t>(rk_block<NT>(tid, j));
    if (need_eq > 0) {
        if (n_eq == need_eq) {
            // every tie is taken: any order (the ranking orders them by id)
            int pe = n_gt + static_cast<int>(ex >> 16);
#pragma unroll
            for (int j = 0; j < PER; ++j)
                if (kk[j] == T)
                    cand[pe++] = (static_cast<unsigned long long>(~kk[j]) << 32) | static_cast<uint32_t>(rk_block<NT>(tid, j));
        } else {
            // more ties than places: the lowest block ids, one row of 4 * NT
            // blocks at a time (within a row, thread order is block order)
            int base = 0;
#pragma unroll
            for (int r = 0; r < PER / 4; ++r) {
                if (base >= need_eq) break;                    // the same for every thread
                int e = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) e += kk[4 * r + k] == T ? 1 : 0;
                int rt;
                int pe = base + group_excl_sum<Grp>(e, sc->tmp, &rt);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int j = 4 * r + k;
                    if (kk[j] == T) {
                        if (pe < need_eq)
                            cand[n_gt + pe] =
                                (static_cast<unsigned long long>(~kk[j]) << 32) | static_cast<uint32_t>(rk_block<NT>(tid, j));
                        ++pe;
                    }
                }
                base += rt;
            }
        }
    }
    for (int i = take + tid; i < kp; i += NT) cand[i] = ~0ull;
    Grp::sync();
    select_finish<Grp>(cand, take, kp, K, s, out, out_s, s_out);
}

// One CTA of kSelThreads per (b, h), keys in registers (nv <= 64 * kSelThreads
// = 32768, the largest block count the library takes).
template <int PER>
__device__ __forceinline__ void select_topk_regs(const float* s, int nv, int K, bool vec4, unsigned long long* cand,
                                                 SelScratch* sc, int32_t* out, float* out_s) {
    using Grp = CtaGroup<kSelThreads>;
    uint32_t kk[PER];
    rk_load_scores<Grp, PER>(kk, s, nv, vec4);
    select_unit_regs<Grp, PER>(kk, nv, K, cand, sc, s, out, out_s, nullptr);
}

__global__ void __launch_bounds__(kSelThreads) select_topk_kernel(Dims d, const float* __restrict__ scores,
                                                                  const int32_t* __restrict__ ctx_len,
                                                                  int32_t* __restrict__ sel,
                                                                  float* __restrict__ sel_score) {
    __shared__ __align__(16) unsigned long long cand[kSelMaxK];
    __shared__ SelScratch sc;
    const int bh = blockIdx.x, b = bh / d.Hkv;
    const int nv = n_valid_blocks(ctx_len[b], d.N);
    const float* s = scores + static_cast<long long>(bh) * d.N;
    const bool vec4 = (d.N & 3) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15) == 0;
    int32_t* out = sel + static_cast<long long>(bh) * d.K;
    float* out_s = sel_score ? sel_score + static_cast<long long>(bh) * d.K : nullptr;
    if (nv <= 4 * kSelThreads)
        select_topk_regs<4>(s, nv, d.K, vec4, cand, &sc, out, out_s);
    else if (nv <= 16 * kSelThreads)
        select_topk_regs<16>(s, nv, d.K, vec4, cand, &sc, out, out_s);
    else
        select_topk_regs<64>(s, nv, d.K, vec4, cand, &sc, out, out_s);
}

}  // namespace oasis
