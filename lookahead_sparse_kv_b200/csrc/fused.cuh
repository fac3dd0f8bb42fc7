// fused.cuh - lookahead scores, top-K selection and the capped fetch plan in
// one launch.
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching, Figure 8: per layer the drafts drive the top-K prediction,
// the prediction is diffed against the resident blocks, and only then can
// the transfer start, so the three steps sit back to back on the path to the
// copy; method sketch item 4.
//
// The grid is the scorer's: one CTA per 128-block tile of each (b, h) unit
// (lookahead_score_kernel's tile, on the tensor cores).  After writing its
// scores a CTA takes a ticket on the unit's counter; the CTA that completes
// the unit (the last of its ceil(valid blocks / 128) tiles to finish) reads
// all of the unit's scores back from L2 and runs the top-K selection and the
// plan of the unit in its tail, then resets the counter.  No CTA waits for
// another: the selection and the plan of a unit overlap the scoring of the
// others, and the two separate launches (and their serial latency) are gone.
// The results are those of the three separate kernels bit for bit: the same
// scores, select_unit and plan_unit.
#pragma once

#include "common.cuh"
#include "plan.cuh"
#include "score.cuh"
#include "select.cuh"

namespace oasis {

// Shared memory of the fused tail: keys [N] u32, candidates
// [next_pow2(min(K, N))] u64, plan scratch.
__host__ __device__ inline int fused_tail_bytes(int N, int K) {
    int kp = 1;
    while (kp < (K < N ? K : N)) kp <<= 1;
    return ((N * 4 + 7) / 8) * 8 + kp * 8 + plan_smem_ints(K) * 4;
}

// slot_table == NULL: scores and selection only (no plan).  kScored: victims
// by the block's score (read from `scores`), else LRU.  step_dev (nullable):
// the step number is read from device memory.
template <int NPAD, bool kScored>
__global__ void __launch_bounds__(128) score_select_plan_kernel(
    const __grid_constant__ CUtensorMap tm_kmax, const __grid_constant__ CUtensorMap tm_kmin, Dims d,
    const uint16_t* __restrict__ q, const int32_t* __restrict__ ctx_len, float* scores, int row0, int rows,
    int* ticket, int32_t* sel, float* sel_score, int32_t* slot_table, int32_t* last_used, int step,
    const int32_t* __restrict__ step_dev, int32_t* fetch_slot, int32_t* fetch_block, int32_t* n_fetch) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ SelScratch sc;
    __shared__ int tmp[32];
    __shared__ int s_last;
    const int tid = threadIdx.x;
    const int bh = blockIdx.y, b = bh / d.Hkv, h = bh % d.Hkv;
    const int nv = n_valid_blocks(ctx_len[b], d.N);
    const int parts = max(1, (nv + kScoreTile - 1) / kScoreTile);   // CTAs that take a ticket
    if (static_cast<int>(blockIdx.x) >= parts) return;
    const int n0 = blockIdx.x * kScoreTile;
    if (n0 < nv) score_tile<NPAD>(&tm_kmax, &tm_kmin, d, q, b, h, n0, nv, scores, row0, rows, smem);

    // the CTA that finishes the unit selects and plans it
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(ticket + bh, 1) == parts - 1 ? 1 : 0;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (tid == 0) ticket[bh] = 0;                                     // ready for the next call
    const int N = d.N, K = d.K;
    const float* su = scores + static_cast<long long>(bh) * N;
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem);
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(smem + ((N * 4 + 7) / 8) * 8);
    int kp = 1;
    while (kp < min(K, N)) kp <<= 1;
    int32_t* sp = reinterpret_cast<int32_t*>(cand + kp);
    for (int i = tid; i < nv; i += 128) keys[i] = ordered_key(__ldcg(su + i));
    __syncthreads();
    int32_t* sel_u = sel + static_cast<long long>(bh) * K;
    select_unit<128>(keys, nv, K, cand, &sc, su, sel_u, sel_score ? sel_score + static_cast<long long>(bh) * K : nullptr);
    if (slot_table == nullptr) return;
    __syncthreads();                                                  // the selection is in memory
    if (step_dev != nullptr) step = *step_dev;
    plan_unit<128, kScored>(K, d.C, N, sel_u, kScored ? su : nullptr, slot_table + static_cast<long long>(bh) * K,
                            last_used + static_cast<long long>(bh) * K, step,
                            fetch_slot + static_cast<long long>(bh) * d.C, fetch_block + static_cast<long long>(bh) * d.C,
                            n_fetch + bh, sp, tmp);
}

}  // namespace oasis
