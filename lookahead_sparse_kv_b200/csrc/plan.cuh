// plan.cuh - residency diff, capped fetch list and LRU victims.
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching: method sketch item 3 (the prediction is diffed against the
// GPU-resident blocks; only the difference is copied, under a per-step cap),
// Table 2 (LRU eviction), Figure 9 (a per-KV-head table maps each GPU
// block slot to a CPU block), "Terms in this paper" (capped eviction).
//
// One group of threads per (b, h), each thread looping over slots / ranks
// (K <= 1024):
//   1. the resident blocks go into a hash table in shared memory (block id ->
//      lowest slot holding it; a second slot with the same block is an
//      error); each selected block looks itself up there, and hits protect
//      their slot and stamp it with the step;
//   2. misses are numbered in rank order by a group-wide scan; the first
//      min(C, |M|) are fetched;
//   3. every unprotected slot j has a 64-bit victim key - free slots (0, j),
//      stale slots (1, order, block id) - and its rank among the candidates
//      by counting smaller keys; rank r < nF receives fetch r.
//      order = last_used (LRU, Table 2) or, for the score-based variant of
//      the eviction ablation, the block's current lookahead score mapped to
//      a monotone integer key (lowest score evicted first).
// Integer only (the score enters as its order key), so the result is
// bit-exact against any correct planner.
#pragma once

#include "common.cuh"

namespace oasis {

// order: an unsigned key, smaller = evicted earlier (blk < 15 bits, N <= 32768)
__device__ __forceinline__ unsigned long long victim_key(int slot, int blk, uint32_t order) {
    if (blk < 0) return static_cast<unsigned long long>(slot);
    return (1ull << 63) | (static_cast<unsigned long long>(order) << 31) |
           static_cast<unsigned long long>(static_cast<uint32_t>(blk));
}

constexpr int kPlanThreads = 256;

// Shared-memory layout of plan_unit for budget K, in ints: eight arrays of K
// rounded up to a multiple of 4 (so the scans over slots read 16 B at a
// time), the victim keys (64-bit, same count) and the hash table (2 entries
// per slot, a power of two).
__host__ __device__ constexpr int plan_k4(int K) { return (K + 3) & ~3; }
__host__ __device__ constexpr int plan_pow2(int K) { return K <= 1 ? 1 : 2 * plan_pow2((K + 1) / 2); }
__host__ __device__ constexpr int plan_hash_size(int K) { return K <= 2 ? 4 : 2 * plan_pow2(K); }   // >= 4: 16-B multiple
__host__ __device__ constexpr int plan_smem_ints(int K) { return 10 * plan_k4(K) + plan_hash_size(K); }
// The selection's place in that layout: a caller may write the selection
// there itself and pass this pointer as `sel`.
__device__ __forceinline__ int32_t* plan_sel_smem(int32_t* sp, int K) { return sp + 6 * plan_k4(K); }

// Starts copying a unit's slot table and recency into the plan's shared
// memory (each thread its slots tid, tid + NT, ...), for plan_unit(...,
// staged = true) to use once they have landed.
template <class Grp>
__device__ __forceinline__ void plan_stage_async(int K, const int32_t* st, const int32_t* lu, int32_t* sp) {
    const int K4 = plan_k4(K);
    for (int i = Grp::tid(); i < K; i += Grp::kThreads) {
        cp_async_4(sp + i, st + i);
        cp_async_4(sp + K4 + i, lu + i);
    }
    cp_async_commit();
}

constexpr uint32_t kPlanHashEmpty = 0xFFFFFFFFu;
__device__ __forceinline__ uint32_t plan_hash(uint32_t blk, int log2_size) {
    return (blk * 0x9E3779B1u) >> (32 - log2_size);
}

// Plan of one (b, h) by a group of threads (each loops over slots /
// ranks): sel, st, lu point at the unit's K entries, fs/fb at its C fetch
// entries, nf at its fetch count; scores_u (kScored) at its N block scores.
// sp: plan_smem_ints(K) ints of shared memory, 16-B aligned; tmp: 32 ints.
// staged: the caller has already copied st and lu into the first two arrays
// of sp (plan_stage_async, each thread its own slots tid, tid + NT, ...).
template <class Grp, bool kScored>
__device__ void plan_unit(int K, int C, int N, const int32_t* sel, const float* scores_u, int32_t* st, int32_t* lu,
                          int step, int32_t* fs, int32_t* fb, int32_t* nf, int32_t* sp, int* tmp,
                          bool staged = false) {
    constexpr int NT = Grp::kThreads;
    const int K4 = plan_k4(K);
    int32_t* s_st = sp;
    int32_t* s_lu = sp + K4;
    int32_t* s_prot = sp + 2 * K4;
    int32_t* s_vict = sp + 3 * K4;
    int32_t* s_nst = sp + 4 * K4;
    int32_t* s_nlu = sp + 5 * K4;
    int32_t* s_sel = sp + 6 * K4;          // == plan_sel_smem(sp, K)
    int32_t* s_mpos = sp + 7 * K4;         // miss flag, then the miss's position in rank order (-1: no miss)
    unsigned long long* s_vk = reinterpret_cast<unsigned long long*>(sp + 8 * K4);   // victim keys, ~0: not a victim
    uint32_t* s_hash = reinterpret_cast<uint32_t*>(sp + 10 * K4);
    const int hs = plan_hash_size(K), hlog = __ffs(hs) - 1;
    const int tid = Grp::tid();
    for (int i = K + tid; i < K4; i += NT) {   // padding: never matches, never a victim
        s_st[i] = -2;
        s_prot[i] = 1;
        s_vk[i] = ~0ull;
    }
    for (int i = tid; i < hs; i += NT) s_hash[i] = kPlanHashEmpty;
    const bool sel_here = sel == s_sel;
    auto stage = [&](int i, int x, int l) {
        if (x < -1 || x >= N) {
            raise_dev_error(OASIS_DEVERR_ID_RANGE);
            x = -1;
        }
        s_st[i] = x;
        s_lu[i] = l;
        s_prot[i] = 0;
        uint32_t ord;
        if constexpr (kScored)
            ord = x >= 0 ? ordered_key(__ldcg(scores_u + x)) : 0u;
        else
            ord = static_cast<uint32_t>(l) ^ 0x80000000u;   // signed order
        s_vk[i] = victim_key(i, x, ord);
        if (!sel_here) {
            int sv = sel[i];
            if (sv < -1 || sv >= N) {
                raise_dev_error(OASIS_DEVERR_ID_RANGE);
                sv = -1;
            }
            s_sel[i] = sv;
        }
    };
    if (staged) {
        cp_async_wait_all();                 // this thread's own copies have landed
        for (int i = tid; i < K; i += NT) stage(i, s_st[i], s_lu[i]);
    } else {
        for (int i = tid; i < K; i += NT) stage(i, st[i], lu[i]);
    }
    Grp::sync();
    // 1a. resident blocks into the table: entry (block << 10 | slot); a block
    //     found there already is resident twice (the lower slot is kept)
    for (int i = tid; i < K; i += NT) {
        const int x = s_st[i];
        if (x < 0) continue;
        const uint32_t e = (static_cast<uint32_t>(x) << 10) | static_cast<uint32_t>(i);
        uint32_t pos = plan_hash(static_cast<uint32_t>(x), hlog);
        for (int probe = 0; probe < hs; ++probe) {
            const uint32_t old = atomicCAS(s_hash + pos, kPlanHashEmpty, e);
            if (old == kPlanHashEmpty) break;
            if ((old >> 10) == static_cast<uint32_t>(x)) {
                raise_dev_error(OASIS_DEVERR_DUPLICATE);
                atomicMin(s_hash + pos, e);
                break;
            }
            pos = (pos + 1) & (hs - 1);
        }
    }
    Grp::sync();
    // 1b. residency lookup of every selected block (hits are protected)
    for (int i = tid; i < K; i += NT) {
        const int sv = s_sel[i];
        int hit = -1;
        if (sv >= 0) {
            uint32_t pos = plan_hash(static_cast<uint32_t>(sv), hlog);
            for (int probe = 0; probe < hs; ++probe) {
                const uint32_t e = s_hash[pos];
                if (e == kPlanHashEmpty) break;
                if ((e >> 10) == static_cast<uint32_t>(sv)) {
                    hit = static_cast<int>(e & 1023u);
                    break;
                }
                pos = (pos + 1) & (hs - 1);
            }
        }
        if (hit >= 0) {
            s_prot[hit] = 1;
            s_vk[hit] = ~0ull;
        }
        s_mpos[i] = (sv >= 0 && hit < 0) ? 1 : 0;
    }
    Grp::sync();
    // 2. misses numbered in rank order
    int running = 0;
    for (int base = 0; base < K; base += NT) {
        const int i = base + tid;
        const int m = i < K ? s_mpos[i] : 0;
        int total;
        const int excl = group_excl_sum<Grp>(m, tmp, &total);     // syncs
        if (i < K) s_mpos[i] = m ? running + excl : -1;
        running += total;
    }
    const int nF = min(C, running);
    // 3. victims: rank of every unprotected slot among the candidates
    for (int i = tid; i < K; i += NT) {
        const bool prot = s_prot[i] != 0;
        s_nst[i] = s_st[i];
        s_nlu[i] = prot ? step : s_lu[i];
        if (!prot && nF > 0) {
            const unsigned long long mine = s_vk[i];
            const ulonglong2* vk2 = reinterpret_cast<const ulonglong2*>(s_vk);
            int r0 = 0, r1 = 0;
#pragma unroll 4
            for (int j2 = 0; j2 < K4 / 2; j2 += 2) {
                const ulonglong2 x = vk2[j2], y = vk2[j2 + 1];
                r0 += (x.x < mine) + (x.y < mine);
                r1 += (y.x < mine) + (y.y < mine);
            }
            const int rank = r0 + r1;
            if (rank < nF) s_vict[rank] = i;
        }
    }
    Grp::sync();
    // 4. the first nF misses replace the victims in order
    for (int i = tid; i < K; i += NT) {
        const int mp = s_mpos[i];
        if (mp >= 0 && mp < nF) {
            const int v = s_vict[mp];
            s_nst[v] = s_sel[i];
            s_nlu[v] = step;
            fs[mp] = v;
            fb[mp] = s_sel[i];
        }
    }
    Grp::sync();
    for (int i = tid; i < K; i += NT) {
        st[i] = s_nst[i];
        lu[i] = s_nlu[i];
    }
    for (int f = nF + tid; f < C; f += NT) {
        fs[f] = -1;
        fb[f] = -1;
    }
    if (tid == 0) *nf = nF;
}

// One CTA of kPlanThreads per (b, h); dynamic smem plan_smem_ints(K) ints.
// kScored: victims by the block's score (scores fp32 [B][Hkv][N]), else LRU.
// step_dev (nullable): the step number is read from device memory instead of
// `step`, so a captured graph can replay the plan at every step.
template <bool kScored>
__global__ void __launch_bounds__(kPlanThreads) plan_fetch_kernel(Dims d, const int32_t* __restrict__ sel,
                                                                  const float* __restrict__ scores,
                                                                  int32_t* __restrict__ slot_table,
                                                                  int32_t* __restrict__ last_used, int step,
                                                                  const int32_t* __restrict__ step_dev,
                                                                  int32_t* __restrict__ fetch_slot,
                                                                  int32_t* __restrict__ fetch_block,
                                                                  int32_t* __restrict__ n_fetch) {
    extern __shared__ int32_t sp[];
    __shared__ int tmp[32];
    const long long bh = blockIdx.x;
    const long long base = bh * d.K;
    if (step_dev != nullptr) step = *step_dev;
    plan_unit<CtaGroup<kPlanThreads>, kScored>(d.K, d.C, d.N, sel + base, kScored ? scores + bh * d.N : nullptr,
                                     slot_table + base, last_used + base, step, fetch_slot + bh * d.C,
                                     fetch_block + bh * d.C, n_fetch + bh, sp, tmp);
}

// Residency loss: frees every slot whose mask byte is set (n = B*Hkv*K).
__global__ void evict_slots_kernel(long long n, const uint8_t* __restrict__ mask, int32_t* __restrict__ slot_table) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x)
        if (mask[i]) slot_table[i] = -1;
}

// Advances a device-resident step counter by one (one thread).
__global__ void step_advance_kernel(int32_t* step) { *step += 1; }

}  // namespace oasis
