// fused.cuh - lookahead scores, top-K selection and the capped fetch plan in
// one persistent launch.
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching, Figure 8: per layer the drafts drive the top-K prediction,
// the prediction is diffed against the resident blocks, and only then can
// the transfer start, so the three steps sit back to back on the path to the
// copy; method sketch item 4.  The per-block bound is Quest's (Quest:
// Query-Aware Sparsity for Efficient Long-Context LLM Inference), computed on
// the tensor cores as in score.cuh: for 128 blocks and the R = draft rows x G
// query vectors of a (sequence, KV head) unit,
//     S[128 x R] = [kmax | kmin][128 x 256] . [q+ | q-]^T[256 x R].
//
// Work split: a unit's ceil(N / 128) block tiles are cut into chunks of `cts`
// tiles; CTAs (at most one per SM) take chunks from an atomic counter in
// unit-major order, skipping chunks past the unit's context, so units finish
// one after another through the launch and a CTA slowed down by a neighbour
// on its SM simply takes fewer chunks.  Warps are specialised:
//   warp 0    producer: takes a chunk, streams its 64 KiB summary tiles
//             through a 2-stage TMA ring, and TMA-loads the unit's query
//             rows into the operand buffer (double buffered when it fits),
//             where it splits them into [q+ | q-] in place;
//   warp 1    one thread issues the 16 tcgen05.mma of each tile into one of
//             two TMEM accumulators;
//   warps 2-5 read the accumulators back (one TMEM lane quadrant each: 32
//             blocks per warp), take the max over the real columns and store
//             the fp32 scores;
//   warps 6-9 run the top-K selection and the plan of a unit once all of it
//             is scored, while the other warps score on.
// Two ways a unit reaches the selection:
//   - whole units (a chunk covers a unit; the host picks this with at least
//     half as many units as SMs, else about two chunks per SM): the
//     epilogue also keeps the unit's keys in shared memory and hands them to
//     the CTA's own selection warps (an mbarrier each way), which read them
//     into registers;
//   - split units: after a chunk the epilogue adds one to the unit's ticket;
//     the selection warps claim units in order from a second counter (so
//     every CTA selects about B*Hkv / CTAs units, whichever CTAs scored them),
//     wait until the unit's ticket shows all its chunks scored and read its
//     scores from L2 into registers.
// The selection runs on keys in registers (select_unit_regs) up to 64 keys a
// thread (N <= 8192), else on keys in shared memory (select_unit).
// Results are those of the separate lookahead_score / select_topk / plan
// kernels bit for bit (the same MMA, the same selection rule and plan_unit).
// The last CTA to exit resets the counters for the next call.
#pragma once

#include "common.cuh"
#include "plan.cuh"
#include "score.cuh"
#include "select.cuh"

namespace oasis {

constexpr int kSspThreads = 320;                           // 10 warps
constexpr int kSspStages = 2;                              // summary-tile ring
constexpr int kSspTileBytes = kScoreABytes;                // 64 KiB: kmax lo/hi, kmin lo/hi
constexpr int kSspInfoInts = 8;                            // per chunk: end, u, nv, t0, ts, vt
using SspTailGroup = WarpGroup<128, 2, 192>;               // warps 6-9
using SspEpiGroup = WarpGroup<128, 1, 64>;                 // warps 2-5

// barrier indices
constexpr int kSspFull = 0;       // [2] tile landed
constexpr int kSspEmpty = 2;      // [2] tile consumed by its MMAs
constexpr int kSspAccFull = 4;    // [2] accumulator written
constexpr int kSspAccFree = 6;    // [2] accumulator read (4 epilogue warps)
constexpr int kSspBFull = 8;      // [2] unit operand built
constexpr int kSspBFree = 10;     // [2] unit operand no longer read
constexpr int kSspQFull = 12;     // [2] unit's query rows landed in the operand buffer
constexpr int kSspCFull = 14;     // [2] chunk description written (producer)
constexpr int kSspCFree = 16;     // [2] description read (MMA issuer, epilogue leader)
constexpr int kSspFinal = 18;
constexpr int kSspKFull = 19;     // whole units: the unit's keys are in shared memory (epilogue leader)
constexpr int kSspKFree = 20;     // whole units: the selection warps have read them
constexpr int kSspNumBars = 21;
constexpr uint32_t kSspNbEpiVote = 3;                      // named barrier of the epilogue's stop vote

// Chunking of the scoring work (host and device agree through these).
struct SspChunks {
    int cts;     // tiles per chunk
    int cpu;     // chunks per unit (ceil(ceil(N / 128) / cts))
    int nc;      // chunks in all
    int whole;   // cts covers every unit (cpu == 1): keys handed over in shared memory
};
constexpr int kSspRegKeys = 64;                            // keys a tail thread holds in registers at most

template <int NPAD>
struct SspSmem {
    static constexpr int kBBytes = 4 * NPAD * 128;                     // q+ lo/hi, q- lo/hi
    static constexpr int kOffB = kSspStages * kSspTileBytes;
    static constexpr int kOffBar(int nbuf) { return kOffB + nbuf * kBBytes; }
    static constexpr int kOffMisc(int nbuf) { return kOffBar(nbuf) + kSspNumBars * 8; }   // 64 ints
    static constexpr int kOffCand(int nbuf) { return (kOffMisc(nbuf) + 256 + 15) / 16 * 16; }
    static constexpr int kAccStride = NPAD <= 16 ? 16 : (NPAD <= 32 ? 32 : 64);   // TMEM columns per accumulator
    static constexpr int kTmemCols = 2 * kAccStride < 32 ? 32 : 2 * kAccStride;
    // total dynamic bytes for nbuf operand buffers, budget K and N blocks
    // (candidates, plan scratch, the unit's keys rounded up to 4; +1024
    // alignment slack)
    static constexpr int bytes(int nbuf, int K, int N) {
        int kp = 2;                                  // >= 2 keeps the plan scratch 16-B aligned
        while (kp < K) kp <<= 1;
        return kOffCand(nbuf) + kp * 8 + plan_smem_ints(K) * 4 + ((N + 3) & ~3) * 4 + 1024;
    }
};

// The i-th tile a chunk of nt tiles starting at t0 of unit u takes: the
// chunk's tiles rotated by a unit-dependent amount.
__device__ __forceinline__ int ssp_tile(int u, int t0, int nt, int i) {
    const int r = i + (u * 7) % nt;
    return t0 + (r >= nt ? r - nt : r);
}

// Selection of one unit by the tail warps with PER keys a thread in
// registers, read from the handed-over keys in shared memory (whole units;
// kfree is then arrived once they are read) or from the scores in L2.
template <int PER>
__device__ __forceinline__ void ssp_select_regs(bool from_smem, const uint32_t* keys, const float* su, bool vec4, int nv,
                                                int K, unsigned long long* cand, SelScratch* sc, int32_t* sel_u,
                                                float* ss_u, int32_t* s_sel, uint64_t* kfree) {
    uint32_t kk[PER];
    if (from_smem)
        rk_load_keys<SspTailGroup, PER>(kk, keys, nv);
    else
        rk_load_scores<SspTailGroup, PER>(kk, su, nv, vec4);
    if (kfree) {
        SspTailGroup::sync();                                  // every thread has its keys
        if (SspTailGroup::tid() == 0) mbar_arrive(kfree);
    }
    select_unit_regs<SspTailGroup, PER>(kk, nv, K, cand, sc, su, sel_u, ss_u, s_sel);
}

template <int NPAD, bool kScored>
__global__ void __launch_bounds__(kSspThreads, 1) score_select_plan_kernel(
    const __grid_constant__ CUtensorMap tm_kmax, const __grid_constant__ CUtensorMap tm_kmin,
    const __grid_constant__ CUtensorMap tm_q, Dims d,
    const uint16_t* __restrict__ q, const int32_t* __restrict__ ctx_len, float* scores, int row0, int rows,
    int* ticket, int* sched, int32_t* sel, float* sel_score, int32_t* slot_table, int32_t* last_used, int step,
    const int32_t* __restrict__ step_dev, int32_t* fetch_slot, int32_t* fetch_block, int32_t* n_fetch,
    SspChunks ch, int nbuf) {
    using S = SspSmem<NPAD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ SelScratch sc;
    __shared__ int tmp[32];
    uint8_t* ring = smem;
    uint8_t* bbuf = smem + S::kOffB;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + S::kOffBar(nbuf));
    int* misc = reinterpret_cast<int*>(smem + S::kOffMisc(nbuf));
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(misc);
    volatile int* s_abort = misc + 1;
    int* s_info = misc + 8;                               // [2][kSspInfoInts] chunk descriptions
    volatile int* s_claim = misc + 24;                    // the tail group's claimed unit
    volatile int* s_kunit = misc + 25;                    // whole units: the unit whose keys are handed over
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(smem + S::kOffCand(nbuf));
    int kp = 2;
    while (kp < d.K) kp <<= 1;
    int32_t* sp = reinterpret_cast<int32_t*>(cand + kp);   // 16-B aligned
    uint32_t* keys = reinterpret_cast<uint32_t*>(sp + plan_smem_ints(d.K));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long N = d.N;

    if (tid == 0) {
        for (int i = 0; i < kSspNumBars; ++i)
            mbar_init(&bar[i], (i == kSspAccFree || i == kSspAccFree + 1) ? 4
                               : (i == kSspCFree || i == kSspCFree + 1) ? 2
                                                                         : 1);   // KFull, KFree: 1
        fence_mbar_init();
        *s_abort = 0;
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, S::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *s_tmem;
    const int G = d.G();

    if (warp == 0) {
        // ========================================================= producer
        if (lane == 0) {
            prefetch_tensormap(&tm_kmax);
            prefetch_tensormap(&tm_kmin);
            prefetch_tensormap(&tm_q);
        }
        const uint64_t pol = l2_policy_evict_first();
        const uint64_t pol_q = l2_policy_evict_last();
        int pos = 0, nb = 0;
        int last_pos[kSspStages] = {-1, -1};
        // tile t of unit u into the ring (lane 0)
        auto load_tile = [&](int u, int t) {
            const int stage = pos % kSspStages;
            if (pos >= kSspStages) cta_wait(&bar[kSspEmpty + stage], ((pos / kSspStages) - 1) & 1, s_abort);
            mbar_arrive_expect_tx(&bar[kSspFull + stage], kSspTileBytes);
            if (!*s_abort) {
                last_pos[stage] = pos;
                uint8_t* st = ring + stage * kSspTileBytes;
                const int y = static_cast<int>(u * N + t * kScoreTile);
                tma_load_2d(st + 0 * kScoreRegionBytes, &tm_kmax, &bar[kSspFull + stage], 0, y, pol);
                tma_load_2d(st + 1 * kScoreRegionBytes, &tm_kmax, &bar[kSspFull + stage], 64, y, pol);
                tma_load_2d(st + 2 * kScoreRegionBytes, &tm_kmin, &bar[kSspFull + stage], 0, y, pol);
                tma_load_2d(st + 3 * kScoreRegionBytes, &tm_kmin, &bar[kSspFull + stage], 64, y, pol);
            }
            ++pos;
        };
        // requested one chunk ahead: the first is the CTA's block index (grid <=
        // chunks), the rest come from the counter, numbered from the grid size on
        int c_next = static_cast<int>(blockIdx.x);
        for (int p = 0;; ++p) {
            const int pb = p & 1;
            int* info = s_info + pb * kSspInfoInts;
            if (lane == 0 && p >= 2) cta_wait(&bar[kSspCFree + pb], ((p >> 1) - 1) & 1, s_abort);
            // the next chunk that holds valid blocks (every unit has one: its chunk 0)
            int u = 0, nv = 0, t0 = 0, vt = 0, c = 0;
            while (true) {
                if (lane == 0) {
                    c = *s_abort ? ch.nc : c_next;
                    if (c < ch.nc) c_next = static_cast<int>(gridDim.x) + atomicAdd(sched, 1);
                }
                c = __shfl_sync(0xFFFFFFFFu, c, 0);
                if (c >= ch.nc) break;
                u = c / ch.cpu;
                t0 = (c - u * ch.cpu) * ch.cts;
                nv = n_valid_blocks(ctx_len[u / d.Hkv], d.N);
                vt = max(1, (nv + kScoreTile - 1) / kScoreTile);
                if (t0 < vt) break;
            }
            if (c >= ch.nc) {
                if (lane == 0) {
                    info[0] = 1;
                    mbar_arrive(&bar[kSspCFull + pb]);
                }
                break;
            }
            const int ts = min(t0 + ch.cts, (nv + kScoreTile - 1) / kScoreTile);   // scored tiles [t0, ts)
            // the chunk's tiles are taken in a rotated order (ssp_tile), so CTAs that
            // start together read different offsets of their units
            const int nt = ts - t0;
            // as many tiles as the ring holds go out first: they wait only on earlier
            // chunks' products; the rest wait on this chunk's, so the operand comes first
            const int n_pre = min(nt, kSspStages);
            if (lane == 0) {
                info[0] = 0;
                info[1] = u;
                info[2] = nv;
                info[3] = t0;
                info[4] = ts;
                info[5] = vt;
                mbar_arrive(&bar[kSspCFull + pb]);
                for (int i = 0; i < n_pre; ++i) load_tile(u, ssp_tile(u, t0, nt, i));
            }
            __syncwarp();
            if (ts > t0) {
                // [q+ | q-] of the unit's scored rows in four 64-column regions (128-byte
                // swizzle): the rows land in the q+ regions by TMA, and each 16-B piece is
                // split there, its negative lanes going to the same place in the q- regions
                const int b = u / d.Hkv, h = u - b * d.Hkv;
                const int bb = nb % nbuf;
                uint8_t* bt = bbuf + bb * S::kBBytes;
                if (lane == 0) {
                    if (nb >= nbuf) cta_wait(&bar[kSspBFree + bb], ((nb / nbuf) - 1) & 1, s_abort);
                    mbar_arrive_expect_tx(&bar[kSspQFull + bb], static_cast<uint32_t>(rows) * kRowBytes);
                    if (!*s_abort) {
                        tma_load_3d(bt, &tm_q, &bar[kSspQFull + bb], 0, h * G, b * d.Qn + row0, pol_q);
                        tma_load_3d(bt + NPAD * 128, &tm_q, &bar[kSspQFull + bb], 64, h * G, b * d.Qn + row0, pol_q);
                    }
                }
                __syncwarp();
                cta_wait(&bar[kSspQFull + bb], (nb / nbuf) & 1, s_abort);
                for (int it = lane; it < rows * 16; it += 32) {
                    const int r = it >> 4, cc16 = it & 15;
                    const int region = cc16 >> 3, cc = cc16 & 7;
                    const int off = region * NPAD * 128 + (r >> 3) * 1024 + (r & 7) * 128 + ((cc ^ (r & 7)) << 4);
                    const uint4 v = *reinterpret_cast<const uint4*>(bt + off);
                    uint32_t w[4] = {v.x, v.y, v.z, v.w}, pos4[4], neg4[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t neg_mask = ((w[i] & 0x80008000u) >> 15) * 0xFFFFu;
                        neg4[i] = w[i] & neg_mask;
                        pos4[i] = w[i] & ~neg_mask;
                    }
                    *reinterpret_cast<uint4*>(bt + off) = make_uint4(pos4[0], pos4[1], pos4[2], pos4[3]);
                    *reinterpret_cast<uint4*>(bt + 2 * NPAD * 128 + off) = make_uint4(neg4[0], neg4[1], neg4[2], neg4[3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&bar[kSspBFull + bb]);
                    for (int i = n_pre; i < nt; ++i) load_tile(u, ssp_tile(u, t0, nt, i));
                }
                ++nb;
            }
            __syncwarp();
            pos = __shfl_sync(0xFFFFFFFFu, pos, 0);
        }
        if (lane == 0)                                     // no copy may land after the CTA exits
            for (int s = 0; s < kSspStages; ++s)
                if (last_pos[s] >= 0) mbar_wait(&bar[kSspFull + s], static_cast<uint32_t>((last_pos[s] / kSspStages) & 1));
    } else if (warp == 1) {
        // ======================================================= MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16_f32(kScoreTile, NPAD);
            int pos = 0, nb = 0;
            for (int p = 0;; ++p) {
                const int pb = p & 1;
                if (!cta_wait(&bar[kSspCFull + pb], (p >> 1) & 1, s_abort)) break;
                const int* info = s_info + pb * kSspInfoInts;
                if (info[0]) break;
                const int t0 = info[3], ts = info[4];
                if (ts > t0) {
                    const int bb = nb % nbuf;
                    cta_wait(&bar[kSspBFull + bb], (nb / nbuf) & 1, s_abort);
                    const uint32_t b0 = smem_addr(bbuf + bb * S::kBBytes);
                    for (int t = t0; t < ts; ++t, ++pos) {
                        const int stage = pos % kSspStages;
                        const int ab = pos & 1;
                        bool ok = cta_wait(&bar[kSspFull + stage], (pos / kSspStages) & 1, s_abort);
                        if (pos >= 2) ok = cta_wait(&bar[kSspAccFree + ab], ((pos >> 1) - 1) & 1, s_abort) && ok;
                        tc_fence_after_sync();
                        if (ok) {
                            const uint32_t a0 = smem_addr(ring + stage * kSspTileBytes);
#pragma unroll
                            for (int reg = 0; reg < 4; ++reg)
#pragma unroll
                                for (int ks = 0; ks < 4; ++ks)
                                    umma_bf16(tmem + ab * S::kAccStride,
                                              umma_desc_sw128(a0 + reg * kScoreRegionBytes + ks * 32),
                                              umma_desc_sw128(b0 + reg * NPAD * 128 + ks * 32), idesc,
                                              (reg | ks) != 0);
                        }
                        umma_commit(&bar[kSspAccFull + ab]);
                        umma_commit(&bar[kSspEmpty + stage]);
                    }
                    umma_commit(&bar[kSspBFree + bb]);         // after the chunk's last MMA
                    ++nb;
                }
                mbar_arrive(&bar[kSspCFree + pb]);
            }
            umma_commit(&bar[kSspFinal]);
            mbar_wait(&bar[kSspFinal], 0);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ========================================== score epilogue (2..5)
        const int qd = warp & 3;                               // TMEM lane quadrant = 32 blocks of the tile
        const bool leader = warp == 2 && lane == 0;
        int pos = 0;
        for (int p = 0;; ++p) {
            const int pb = p & 1;
            cta_wait(&bar[kSspCFull + pb], (p >> 1) & 1, s_abort);
            const int* info = s_info + pb * kSspInfoInts;
            const int end = info[0], u = info[1], nv = info[2], t0 = info[3], ts = info[4];
            // whole units: the previous unit's keys must have been read before
            // this unit's (or the end mark) go into shared memory
            if (ch.whole && p > 0) cta_wait(&bar[kSspKFree], (p - 1) & 1, s_abort);
            if (named_bar_or(kSspNbEpiVote, 128, end != 0 || *s_abort)) {
                if (ch.whole && leader) {
                    *s_kunit = -1;
                    mbar_arrive(&bar[kSspKFull]);
                }
                break;
            }
            for (int i = 0; i < ts - t0; ++i, ++pos) {
                const int t = ssp_tile(u, t0, ts - t0, i);
                const int ab = pos & 1;
                const bool ok = cta_wait(&bar[kSspAccFull + ab], (pos >> 1) & 1, s_abort);
                __syncwarp();                                      // tcgen05.ld is warp-wide: lanes together
                tc_fence_after_sync();
                float best = -__int_as_float(0x7f800000);
                if (ok) {
#pragma unroll
                    for (int c0 = 0; c0 < NPAD; c0 += 16) {
                        uint32_t v[16];
                        tmem_ld_x16(tmem + (static_cast<uint32_t>(qd * 32) << 16) + ab * S::kAccStride + c0, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < rows) best = fmaxf(best, __uint_as_float(v[i]));
                    }
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar[kSspAccFree + ab]);
                const int n = t * kScoreTile + qd * 32 + lane;
                if (ok && n < nv) {
                    scores[u * N + n] = best;
                    if (ch.whole) keys[n] = ordered_key(best);
                }
            }
            if (ch.whole) {
                // the unit's keys (and scores) are out: hand them to the selection warps
                SspEpiGroup::sync();
                if (leader) {
                    *s_kunit = u;
                    mbar_arrive(&bar[kSspKFull]);
                    mbar_arrive(&bar[kSspCFree + pb]);
                }
            } else {
                // the chunk's scores are out: one more chunk of the unit done
                __threadfence();
                SspEpiGroup::sync();
                if (leader) {
                    atomicAdd(ticket + u, 1);
                    mbar_arrive(&bar[kSspCFree + pb]);
                }
            }
        }
    } else {
        // ====================================== top-K + plan tail (6..9)
        const int ttid = SspTailGroup::tid();
        const int units = d.B * d.Hkv;
        const bool vec4 = (N & 3) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15) == 0;
        int32_t* s_sel = slot_table != nullptr ? plan_sel_smem(sp, d.K) : nullptr;
        for (int k = 0;; ++k) {
            int u;
            if (ch.whole) {
                // the next unit this CTA scored (one thread waits, the others at the barrier)
                if (ttid == 0) {
                    bool ok = !*s_abort;
                    if (ok && !mbar_wait_idle(&bar[kSspKFull], k & 1)) {
                        *s_abort = 1;
                        raise_dev_error(OASIS_DEVERR_TIMEOUT);
                        ok = false;
                    }
                    *s_claim = ok ? *s_kunit : -1;
                }
                SspTailGroup::sync();
                u = *s_claim;
                SspTailGroup::sync();
                if (u < 0) break;
            } else {
                // claim the next unit; wait until every chunk of it holding valid blocks is scored
                if (ttid == 0) {
                    int c = *s_abort ? units : atomicAdd(sched + 2, 1);
                    if (c < units) {
                        const int nvu = n_valid_blocks(ctx_len[c / d.Hkv], d.N);
                        const int vt = max(1, (nvu + kScoreTile - 1) / kScoreTile);
                        const int chunks = (vt + ch.cts - 1) / ch.cts;
                        const uint64_t t0 = global_timer_ns();
                        while (ld_acquire_gpu(ticket + c) < chunks) {
                            if (global_timer_ns() - t0 > kWaitLimitNs) {   // bounded: give up, flag it
                                *s_abort = 1;
                                raise_dev_error(OASIS_DEVERR_TIMEOUT);
                                c = units;
                                break;
                            }
                            __nanosleep(64);
                        }
                    }
                    *s_claim = c;
                }
                SspTailGroup::sync();
                u = *s_claim;
                SspTailGroup::sync();
                if (u >= units) break;
                if (ttid == 0) ticket[u] = 0;                  // ready for the next call
            }
            const int nv = n_valid_blocks(ctx_len[u / d.Hkv], d.N);
            const float* su = scores + u * N;
            const long long uk = static_cast<long long>(u) * d.K, uc = static_cast<long long>(u) * d.C;
            // the unit's slot table and recency, copied into the plan's shared
            // memory now (asynchronously) and used by the plan after the selection
            const bool pre = slot_table != nullptr;
            if (pre) plan_stage_async<SspTailGroup>(d.K, slot_table + uk, last_used + uk, sp);
            int32_t* sel_u = sel + static_cast<long long>(u) * d.K;
            float* ss_u = sel_score ? sel_score + static_cast<long long>(u) * d.K : nullptr;
            uint64_t* kfree = ch.whole ? &bar[kSspKFree] : nullptr;
            if (nv <= 16 * SspTailGroup::kThreads) {
                ssp_select_regs<16>(ch.whole != 0, keys, su, vec4, nv, d.K, cand, &sc, sel_u, ss_u, s_sel, kfree);
            } else if (nv <= kSspRegKeys * SspTailGroup::kThreads) {
                ssp_select_regs<kSspRegKeys>(ch.whole != 0, keys, su, vec4, nv, d.K, cand, &sc, sel_u, ss_u, s_sel,
                                             kfree);
            } else {
                // more keys than registers: the unit's keys in shared memory
                if (!ch.whole) {
                    for (int i = ttid; i < nv; i += SspTailGroup::kThreads) keys[i] = ordered_key(__ldcg(su + i));
                    SspTailGroup::sync();
                }
                select_unit<SspTailGroup>(SmemKeys{keys}, nv, d.K, cand, &sc, su, sel_u, ss_u, s_sel);
                if (kfree) {
                    SspTailGroup::sync();                      // keys no longer read
                    if (ttid == 0) mbar_arrive(kfree);
                }
            }
            if (slot_table == nullptr) {
                SspTailGroup::sync();                          // cand / scratch free for the next unit
                continue;
            }
            const int stp = step_dev != nullptr ? *step_dev : step;
            plan_unit<SspTailGroup, kScored>(d.K, d.C, d.N, s_sel, kScored ? su : nullptr, slot_table + uk,
                                             last_used + uk, stp, fetch_slot + uc, fetch_block + uc, n_fetch + u, sp,
                                             tmp, pre);
            SspTailGroup::sync();                              // scratch free for the next unit
        }
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc(tmem, S::kTmemCols);
    if (tid == 0) {
        // the last CTA out resets the chunk counter for the next call
        __threadfence();
        if (atomicAdd(sched + 1, 1) == static_cast<int>(gridDim.x) - 1) {
            atomicExch(sched, 0);
            atomicExch(sched + 2, 0);
            atomicExch(sched + 1, 0);
        }
    }
}

}  // namespace oasis
