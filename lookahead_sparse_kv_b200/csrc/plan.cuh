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

__device__ __forceinline__ int block_excl_sum_any(int v, int* tmp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += n;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xFFFFFFFFu, w, o);
            if (lane >= o) w += n;
        }
        tmp[lane] = w;
    }
    __syncthreads();
    const int incl = x + (warp > 0 ? tmp[warp - 1] : 0);
    *total = tmp[nw - 1];
    __syncthreads();
    return incl - v;
}

// order: an unsigned key, smaller = evicted earlier (blk < 15 bits, N <= 32768)
__device__ __forceinline__ unsigned long long victim_key(int slot, int blk, uint32_t order) {
    if (blk < 0) return static_cast<unsigned long long>(slot);
    return (1ull << 63) | (static_cast<unsigned long long>(order) << 31) |
           static_cast<unsigned long long>(static_cast<uint32_t>(blk));
}

// blockDim.x = K rounded up to a multiple of 32; dynamic smem 7*K ints.
// kScored: victims by the block's score (scores fp32 [B][Hkv][N]), else LRU.
// step_dev (nullable): the step number is read from device memory instead of
// `step`, so a captured graph can replay the plan at every step.
template <bool kScored>
__global__ void __launch_bounds__(1024) plan_fetch_kernel(Dims d, const int32_t* __restrict__ sel,
                                                          const float* __restrict__ scores,
                                                          int32_t* __restrict__ slot_table,
                                                          int32_t* __restrict__ last_used, int step,
                                                          const int32_t* __restrict__ step_dev,
                                                          int32_t* __restrict__ fetch_slot,
                                                          int32_t* __restrict__ fetch_block,
                                                          int32_t* __restrict__ n_fetch) {
    extern __shared__ int32_t sp[];
    const int K = d.K, C = d.C, N = d.N;
    int32_t* s_st = sp;
    int32_t* s_lu = sp + K;
    int32_t* s_prot = sp + 2 * K;
    int32_t* s_vict = sp + 3 * K;
    int32_t* s_nst = sp + 4 * K;
    int32_t* s_nlu = sp + 5 * K;
    uint32_t* s_ord = reinterpret_cast<uint32_t*>(sp + 6 * K);
    __shared__ int tmp[32];

    const int i = threadIdx.x;
    const long long base = static_cast<long long>(blockIdx.x) * K;
    if (step_dev != nullptr) step = *step_dev;
    int sv = -1;
    if (i < K) {
        int st = slot_table[base + i];
        if (st < -1 || st >= N) {
            raise_dev_error(OASIS_DEVERR_ID_RANGE);
            st = -1;
        }
        s_st[i] = st;
        s_lu[i] = last_used[base + i];
        s_prot[i] = 0;
        if constexpr (kScored)
            s_ord[i] = st >= 0 ? ordered_key(scores[static_cast<long long>(blockIdx.x) * N + st]) : 0u;
        else
            s_ord[i] = static_cast<uint32_t>(s_lu[i]) ^ 0x80000000u;   // signed order
        sv = sel[base + i];
        if (sv < -1 || sv >= N) {
            raise_dev_error(OASIS_DEVERR_ID_RANGE);
            sv = -1;
        }
    }
    __syncthreads();

    int hit = -1;
    if (i < K) {
        const int own = s_st[i];
        for (int j = 0; j < K; ++j) {
            const int x = s_st[j];
            if (sv >= 0 && hit < 0 && x == sv) hit = j;
            if (own >= 0 && j < i && x == own) raise_dev_error(OASIS_DEVERR_DUPLICATE);
        }
        if (hit >= 0) s_prot[hit] = 1;
    }
    const int miss = (i < K && sv >= 0 && hit < 0) ? 1 : 0;
    int total_miss;
    const int mpos = block_excl_sum_any(miss, tmp, &total_miss);   // syncs: s_prot visible after
    const int nF = min(C, total_miss);

    if (i < K) {
        const bool prot = s_prot[i] != 0;
        s_nst[i] = s_st[i];
        s_nlu[i] = prot ? step : s_lu[i];
        if (!prot) {
            const unsigned long long mine = victim_key(i, s_st[i], s_ord[i]);
            int rank = 0;
            for (int j = 0; j < K; ++j)
                if (!s_prot[j] && victim_key(j, s_st[j], s_ord[j]) < mine) ++rank;
            if (rank < nF) s_vict[rank] = i;
        }
    }
    __syncthreads();
    if (miss && mpos < nF) {
        const int v = s_vict[mpos];
        s_nst[v] = sv;
        s_nlu[v] = step;
        fetch_slot[static_cast<long long>(blockIdx.x) * C + mpos] = v;
        fetch_block[static_cast<long long>(blockIdx.x) * C + mpos] = sv;
    }
    __syncthreads();
    if (i < K) {
        slot_table[base + i] = s_nst[i];
        last_used[base + i] = s_nlu[i];
    }
    for (int f = nF + i; f < C; f += blockDim.x) {
        fetch_slot[static_cast<long long>(blockIdx.x) * C + f] = -1;
        fetch_block[static_cast<long long>(blockIdx.x) * C + f] = -1;
    }
    if (i == 0) n_fetch[blockIdx.x] = nF;
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
