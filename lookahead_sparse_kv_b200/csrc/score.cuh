// score.cuh - lookahead block scores on the 5th-generation tensor cores.
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching, Figure 7 (right): the drafts are run against the min/max
// compressed keys, and the result ranks the blocks for the next step.  The per-block
// bound is Quest's (Quest: Query-Aware Sparsity for Efficient Long-Context LLM
// Inference): sum_c max(q_c*kmin_c, q_c*kmax_c), maxed over the draft rows
// and the G query heads of the KV head.
//
// Because kmin <= kmax, max(q*kmin, q*kmax) = max(q,0)*kmax + min(q,0)*kmin
// exactly (one of the two products is zero), so for R = draft rows x G query
// vectors the bounds of 128 blocks are one dense contraction
//     S[128 x R] = [kmax | kmin][128 x 256] . [q+ | q-]^T[256 x R]
// with bf16 operands (q+ and q- are exact bf16) and fp32 accumulation.  One
// CTA computes one 128-block tile: TMA brings the tile's kmax/kmin rows into
// 128-byte-swizzled shared memory, the CTA builds q+/q- in the same layout,
// one thread issues 16 tcgen05.mma (K = 16 each) into a TMEM accumulator,
// and each of the 4 warps reads its 32 TMEM lanes (= 32 blocks) and takes
// the max over the R columns in registers.
#pragma once

#include "common.cuh"

namespace oasis {

constexpr int kScoreTile = 128;                           // blocks per CTA = MMA M
constexpr int kScoreRegionBytes = kScoreTile * 128;       // 128 rows x 64 bf16
constexpr int kScoreABytes = 4 * kScoreRegionBytes;       // kmax lo/hi, kmin lo/hi

template <int NPAD>
struct ScoreSmem {
    static constexpr int kBRegion = NPAD * 128;
    static constexpr int kBytes = kScoreABytes + 4 * kBRegion + 64 /*barriers, tmem slot*/ + 1024 /*align*/;
    static constexpr int kTmemCols = NPAD <= 32 ? 32 : (NPAD <= 64 ? 64 : (NPAD <= 128 ? 128 : 256));
};

// Scores of the 128-block tile starting at n0 of unit bh (b, h) into
// scores[bh][n0, nv): called by all 128 threads of the CTA with `smem`
// (1024-aligned, ScoreSmem<NPAD>::kBytes - 1024 bytes).  rows = real query
// vectors (scored query rows x G), the scored rows being row0, row0+1, ...;
// NPAD = rows rounded up to 16.  The shared memory may be reused when it
// returns (its barriers are invalidated).
template <int NPAD>
__device__ __forceinline__ void score_tile(const CUtensorMap* tm_kmax, const CUtensorMap* tm_kmin, const Dims& d,
                                           const uint16_t* __restrict__ q, int b, int h, int n0, int nv,
                                           float* __restrict__ scores, int row0, int rows, uint8_t* smem) {
    using S = ScoreSmem<NPAD>;
    uint8_t* a_tile = smem;
    uint8_t* b_tile = smem + kScoreABytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(b_tile + 4 * S::kBRegion);   // [0] tma full, [1] mma done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
    int* flag = reinterpret_cast<int*>(bars + 3);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = b * d.Hkv + h;

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
        *flag = 0;
    }
    __syncthreads();
    if (tid == 0) {
        const uint64_t pol = l2_policy_evict_first();
        const int y = bh * d.N + n0;
        mbar_arrive_expect_tx(&bars[0], kScoreABytes);
        tma_load_2d(a_tile + 0 * kScoreRegionBytes, tm_kmax, &bars[0], 0, y, pol);
        tma_load_2d(a_tile + 1 * kScoreRegionBytes, tm_kmax, &bars[0], 64, y, pol);
        tma_load_2d(a_tile + 2 * kScoreRegionBytes, tm_kmin, &bars[0], 0, y, pol);
        tma_load_2d(a_tile + 3 * kScoreRegionBytes, tm_kmin, &bars[0], 64, y, pol);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, S::kTmemCols);
        tmem_relinquish();
    }

    // B operand: row r = query vector, 256 K-columns [q+ (128) | q- (128)],
    // four 64-column regions in the swizzled K-major layout.
    const int G = d.G();
    for (int it = tid; it < NPAD * 16; it += 128) {
        const int r = it >> 4, c = it & 15;   // c: 8-channel chunk
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < rows) {
            const int j = row0 + r / G;
            const int g = r % G;
            v = *reinterpret_cast<const uint4*>(
                q + ((static_cast<long long>(b) * d.Qn + j) * d.Hq + h * G + g) * kHeadDim + c * 8);
        }
        uint32_t w[4] = {v.x, v.y, v.z, v.w}, pos[4], neg[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t sgn = w[i] & 0x80008000u;
            const uint32_t neg_mask = (sgn >> 15) * 0xFFFFu;   // 0xFFFF in each half whose sign is set
            neg[i] = w[i] & neg_mask;
            pos[i] = w[i] & ~neg_mask;
        }
        const int region = c >> 3, cc = c & 7;
        const int off = (r >> 3) * 1024 + (r & 7) * 128 + ((cc ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(b_tile + region * S::kBRegion + off) = make_uint4(pos[0], pos[1], pos[2], pos[3]);
        *reinterpret_cast<uint4*>(b_tile + (2 + region) * S::kBRegion + off) =
            make_uint4(neg[0], neg[1], neg[2], neg[3]);
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    bool tma_done = false;
    if (tid == 0) {
        if (mbar_wait(&bars[0], 0)) {
            tma_done = true;
            constexpr uint32_t idesc = umma_idesc_bf16_f32(kScoreTile, NPAD);
            const uint32_t a0 = smem_addr(a_tile), b0 = smem_addr(b_tile);
#pragma unroll
            for (int reg = 0; reg < 4; ++reg)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = umma_desc_sw128(a0 + reg * kScoreRegionBytes + ks * 32);
                    const uint64_t bd = umma_desc_sw128(b0 + reg * S::kBRegion + ks * 32);
                    umma_bf16(tmem, ad, bd, idesc, (reg | ks) != 0);
                }
            umma_commit(&bars[1]);
            *flag = 1;
        } else {
            raise_dev_error(OASIS_DEVERR_TIMEOUT);
        }
    }
    __syncthreads();
    const bool issued = *flag != 0;
    bool done = false;
    if (issued) {
        done = mbar_wait(&bars[1], 0);
        if (!done && lane == 0) raise_dev_error(OASIS_DEVERR_TIMEOUT);
    }
    tc_fence_after_sync();
    if (done) {
        float best = -__int_as_float(0x7f800000);
#pragma unroll
        for (int c0 = 0; c0 < NPAD; c0 += 16) {
            uint32_t v[16];
            tmem_ld_x16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (c0 + i < rows) best = fmaxf(best, __uint_as_float(v[i]));
        }
        const int n = n0 + warp * 32 + lane;
        if (n < nv) scores[static_cast<long long>(bh) * d.N + n] = best;
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, S::kTmemCols);
    if (tid == 0) {
        // a copy that never completed must not land in memory reused below
        if (!tma_done && !mbar_wait(&bars[0], 0)) raise_dev_error(OASIS_DEVERR_TIMEOUT);
        mbar_inval(&bars[0]);
        mbar_inval(&bars[1]);
    }
    __syncthreads();
}

template <int NPAD>
__global__ void __launch_bounds__(128) lookahead_score_kernel(const __grid_constant__ CUtensorMap tm_kmax,
                                                              const __grid_constant__ CUtensorMap tm_kmin,
                                                              Dims d, const uint16_t* __restrict__ q,
                                                              const int32_t* __restrict__ ctx_len,
                                                              float* __restrict__ scores, int row0, int rows) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int bh = blockIdx.y, b = bh / d.Hkv, h = bh % d.Hkv;
    const int nv = n_valid_blocks(ctx_len[b], d.N);
    const int n0 = blockIdx.x * kScoreTile;
    if (n0 >= nv) return;   // whole CTA: tile beyond the sequence's context
    score_tile<NPAD>(&tm_kmax, &tm_kmin, d, q, b, h, n0, nv, scores, row0, rows, smem);
}

}  // namespace oasis
