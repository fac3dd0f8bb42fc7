// plan.cuh - residency diff, capped fetch list and LRU victims.
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching: method sketch item 3 (the prediction is diffed against the
// GPU-resident blocks; only the difference is copied, under a per-step cap),
// Table 2 (LRU eviction), Figure 9 (a per-KV-head table maps each GPU
// block slot to a CPU block), "Terms in this paper" (capped eviction).
//
// One CTA per (b, h) with one thread per slot / rank (K <= 1024):
//   1. thread i looks up sel[i] in the slot table (K compares in smem);
//      hits protect their slot and stamp it with the step;
//   2. misses are numbered in rank order by a block-wide scan; the first
//      min(C, |M|) are fetched;
//   3. every unprotected slot j gets a 64-bit victim key - free slots
//      (0, j), stale slots (1, order, block id) - and its rank among the
//      candidates by counting smaller keys; rank r < nF receives fetch r.
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

// Shared-memory ints plan_unit needs for budget K (nine arrays of K rounded
// up to a multiple of 4, so the scans over slots read 16 B at a time).
__host__ __device__ constexpr int plan_k4(int K) { return (K + 3) & ~3; }
__host__ __device__ constexpr int plan_smem_ints(int K) { return 9 * plan_k4(K); }

// Plan of one (b, h) by a group of threads (each loops over slots /
// ranks): sel, st, lu point at the unit's K entries, fs/fb at its C fetch
// entries, nf at its fetch count; scores_u (kScored) at its N block scores.
// sp: plan_smem_ints(K) ints of shared memory; tmp: 32 ints.
template <class Grp, bool kScored>
__device__ void plan_unit(int K, int C, int N, const int32_t* sel, const float* scores_u, int32_t* st, int32_t* lu,
                          int step, int32_t* fs, int32_t* fb, int32_t* nf, int32_t* sp, int* tmp) {
    constexpr int NT = Grp::kThreads;
    const int K4 = plan_k4(K);
    int32_t* s_st = sp;
    int32_t* s_lu = sp + K4;
    int32_t* s_prot = sp + 2 * K4;
    int32_t* s_vict = sp + 3 * K4;
    int32_t* s_nst = sp + 4 * K4;
    int32_t* s_nlu = sp + 5 * K4;
    uint32_t* s_ord = reinterpret_cast<uint32_t*>(sp + 6 * K4);
    int32_t* s_sel = sp + 7 * K4;
    int32_t* s_mpos = sp + 8 * K4;         // miss flag, then the miss's position in rank order (-1: no miss)
    const int tid = Grp::tid();
    for (int i = K + tid; i < K4; i += NT) {   // padding: never matches, never a victim
        s_st[i] = -2;
        s_prot[i] = 1;
        s_ord[i] = 0u;
    }
    for (int i = tid; i < K; i += NT) {
        int x = st[i];
        if (x < -1 || x >= N) {
            raise_dev_error(OASIS_DEVERR_ID_RANGE);
            x = -1;
        }
        s_st[i] = x;
        s_lu[i] = lu[i];
        s_prot[i] = 0;
        if constexpr (kScored)
            s_ord[i] = x >= 0 ? ordered_key(__ldcg(scores_u + x)) : 0u;
        else
            s_ord[i] = static_cast<uint32_t>(s_lu[i]) ^ 0x80000000u;   // signed order
        int sv = sel[i];
        if (sv < -1 || sv >= N) {
            raise_dev_error(OASIS_DEVERR_ID_RANGE);
            sv = -1;
        }
        s_sel[i] = sv;
    }
    Grp::sync();
    // 1. residency lookup of every selected block (hits are protected), and a
    //    check that no block is resident twice; 4 slots per shared-memory read
    const int4* st4 = reinterpret_cast<const int4*>(s_st);
    for (int i = tid; i < K; i += NT) {
        const int sv = s_sel[i], own = s_st[i];
        int hit = 0x7FFFFFFF;
        bool dup = false;
#pragma unroll 4
        for (int j4 = 0; j4 < K4 / 4; ++j4) {
            const int4 x = st4[j4];
            const int j = 4 * j4;
            if (x.w == sv) hit = min(hit, j + 3);
            if (x.z == sv) hit = min(hit, j + 2);
            if (x.y == sv) hit = min(hit, j + 1);
            if (x.x == sv) hit = min(hit, j);
            dup |= (x.x == own && j < i) | (x.y == own && j + 1 < i) | (x.z == own && j + 2 < i) |
                   (x.w == own && j + 3 < i);
        }
        if (sv < 0) hit = 0x7FFFFFFF;
        if (own >= 0 && dup) raise_dev_error(OASIS_DEVERR_DUPLICATE);
        if (hit != 0x7FFFFFFF) s_prot[hit] = 1;
        s_mpos[i] = (sv >= 0 && hit == 0x7FFFFFFF) ? 1 : 0;
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
            const unsigned long long mine = victim_key(i, s_st[i], s_ord[i]);
            const int4* pr4 = reinterpret_cast<const int4*>(s_prot);
            const uint4* or4 = reinterpret_cast<const uint4*>(s_ord);
            int rank = 0;
#pragma unroll 2
            for (int j4 = 0; j4 < K4 / 4; ++j4) {
                const int4 pr = pr4[j4], x = st4[j4];
                const uint4 od = or4[j4];
                const int j = 4 * j4;
                rank += (!pr.x && victim_key(j, x.x, od.x) < mine) + (!pr.y && victim_key(j + 1, x.y, od.y) < mine) +
                        (!pr.z && victim_key(j + 2, x.z, od.z) < mine) + (!pr.w && victim_key(j + 3, x.w, od.w) < mine);
            }
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
