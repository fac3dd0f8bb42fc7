// attn.cuh - sparse GQA decode attention over the resident pool slots, on
// the 5th-generation tensor cores.
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching, Figure 7 (right): the verification query and the drafts are
// attended in one pass over the resident sparse working set; Figure 9: the
// per-head slot table says which block each pool slot holds.
//
// Work split (stream-K): the T = B*Hkv*K pool slots, in (sequence, KV head,
// slot) order, are cut into NS contiguous ranges, one per CTA (one CTA per
// SM).  A CTA walks its range one (sequence, KV head) "unit" piece at a
// time.  Per piece the producer warp lists the occupied slots (free slots and
// blocks past the context skipped), TMA-loads the unit's query rows, and
// streams the listed slots through a 4-stage ring in tiles of 4 slots (64
// tokens): four 2 KiB boxes per slot (K and V, each as two 64-column halves,
// 128-byte swizzle) so that a tile lands as K[64 tokens][128] and
// V[64 tokens][128] in the layouts the tensor core reads.
//
// Math per tile, with the unit's Qn*G query rows as the MMA M dimension
// (padded to 64; M = 64 puts row r in TMEM lane 32*(r/16) + r%16):
//   S[64 x 64]   = Q[64 x 128] . K^T          8 tcgen05.mma, K-major A and B
//   softmax      4 warps, one per TMEM lane quadrant, each thread owning two
//                query rows of 16 tokens (a quad of threads shares a row):
//                running max (moved only when a tile exceeds it by 2^8, so
//                the accumulator is rarely rescaled), exponentials, row sums
//   P            written to shared memory as a bf16 head plus a bf16
//                remainder (~16 significant bits), 128-byte swizzled
//   O[64 x 128] += P_head . V + P_rest . V    V read MN-major, 4 x 2 MMAs
// S is double-buffered in TMEM (S of tile i+1 runs while tile i's softmax
// does), P double-buffered in shared memory; O stays in TMEM for the whole
// piece.  One thread issues every MMA; mbarriers carry every hand-off, with
// bounded waits.
//
// A unit covered by one CTA is normalised and written directly.  A unit
// split over CTAs: each writes a normalised partial (output, log2-sum-exp),
// then takes a ticket with an atomic counter; the last CTA to arrive merges
// all partials of the unit (they are in L2), writes the output and resets the
// counter for the next call.  No CTA ever waits for another.
#pragma once

#include "common.cuh"

namespace oasis {

constexpr int kAttnTileSlots = 4;                                 // slots per tile
constexpr int kAttnStages = 4;                                    // K/V ring depth
constexpr int kAttnRegion = 64 * 128;                             // 64 rows x 128 B = 8 KiB
constexpr int kAttnStageBytes = 4 * kAttnRegion;                  // K lo, K hi, V lo, V hi
constexpr int kAttnRows = 64;                                     // MMA M
constexpr int kAttnMaxList = 1024;                                // slots of one unit (K <= 1024)
constexpr int kAttnThreads = 192;                                 // producer, MMA, 4 softmax warps
constexpr int kAttnTmemCols = 256;                                // S x 2 (64 columns each) + O (128)
constexpr float kLn2 = 0.6931471805599453f;

constexpr int kAttnOffQ = kAttnStages * kAttnStageBytes;          // 2 buffers x (lo, hi)
constexpr int kAttnOffP = kAttnOffQ + 4 * kAttnRegion;            // 2 buffers x (head, rest)
constexpr int kAttnOffList = kAttnOffP + 4 * kAttnRegion;         // 2 x kAttnMaxList ints
constexpr int kAttnOffBar = kAttnOffList + 2 * kAttnMaxList * 4;
constexpr int kAttnNumBars = 26;
constexpr int kAttnOffMisc = kAttnOffBar + kAttnNumBars * 8;
constexpr int kAttnSmem = kAttnOffMisc + 64 + 1024;              // + alignment slack

// mbarrier indices
constexpr int kBarFull = 0;     // [4]  tile landed (producer expect_tx)
constexpr int kBarEmpty = 4;    // [4]  tile's K and V consumed (MMA commit)
constexpr int kBarSFull = 8;    // [2]  S computed (MMA commit)
constexpr int kBarSFree = 10;   // [2]  S read by the 4 softmax warps
constexpr int kBarPFull = 12;   // [2]  P written by the 4 softmax warps
constexpr int kBarPFree = 14;   // [2]  P consumed (MMA commit after PV)
constexpr int kBarQFull = 16;   // [2]  unit's query rows landed
constexpr int kBarQFree = 18;   // [2]  query rows no longer read (MMA commit)
constexpr int kBarLFull = 20;   // [2]  piece's slot list written (producer)
constexpr int kBarLFree = 22;   // [2]  slot list no longer read (MMA thread + softmax leader)
constexpr int kBarODone = 24;   // the piece's last PV has completed
constexpr int kBarFinal = 25;   // teardown: every MMA issued has completed

// Streams whose ranges touch unit u: [first, last].  Slot s belongs to
// stream floor(s * NS / T), so every stream in between touches u.
__host__ __device__ __forceinline__ void attn_unit_streams(long long u, long long K, long long NS, long long T,
                                                           long long* first, long long* last) {
    *first = (u * K) * NS / T;
    *last = ((u + 1) * K - 1) * NS / T;
}

// Waits unless the CTA has given up; a wait that runs out flags the CTA and
// the device error word.  Returns whether the awaited phase completed.
__device__ __forceinline__ bool attn_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity)) return true;
    *abort_flag = 1;
    raise_dev_error(OASIS_DEVERR_TIMEOUT);
    return false;
}

__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_pool, const __grid_constant__ CUtensorMap tm_q, Dims d,
                       const int32_t* __restrict__ slot_table, const int32_t* __restrict__ ctx_len, float scale_log2,
                       int n_streams, float* __restrict__ out, float* __restrict__ lse_out, float* ws_o,
                       float* ws_lse, int* ws_ticket) {
    const float kNegInf = -__int_as_float(0x7f800000);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint8_t* sQ = smem + kAttnOffQ;
    uint8_t* sP = smem + kAttnOffP;
    int* s_list = reinterpret_cast<int*>(smem + kAttnOffList);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kAttnOffBar);
    int* misc = reinterpret_cast<int*>(smem + kAttnOffMisc);
    int* s_nlist = misc;                                  // [2]
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(misc + 2);
    volatile int* s_abort = misc + 3;
    volatile int* s_last = misc + 4;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long K = d.K;
    const long long T = static_cast<long long>(d.B) * d.Hkv * K;
    const long long gs = blockIdx.x;
    const long long s_begin = (gs * T + n_streams - 1) / n_streams;
    const long long s_end = ((gs + 1) * T + n_streams - 1) / n_streams;
    if (s_begin >= s_end) return;                         // whole CTA: empty range
    const long long u_first = s_begin / K, u_last = (s_end - 1) / K;
    const int G = d.G();
    const int rows = d.Qn * G;

    // ---------------------------------------------------------- set-up
    if (tid == 0) {
        const int counts[kAttnNumBars] = {1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 4, 4, 4, 4, 1, 1,
                                          1, 1, 1, 1, 1, 1, 2, 2, 1, 1};
        for (int i = 0; i < kAttnNumBars; ++i) mbar_init(&bar[i], counts[i]);
        fence_mbar_init();
        *s_abort = 0;
        *s_last = 0;
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, kAttnTmemCols);
        tmem_relinquish();
    }
    // zero Q and P: rows past the real query rows stay zero for the whole call
    for (int i = tid; i < 8 * kAttnRegion / 16; i += kAttnThreads)
        reinterpret_cast<uint4*>(sQ)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *s_tmem;
    const uint32_t tmem_o = tmem + 128;

    if (warp == 0) {
        // ===================================================== producer
        if (lane == 0) {
            prefetch_tensormap(&tm_pool);
            prefetch_tensormap(&tm_q);
        }
        const uint64_t pol_kv = l2_policy_evict_first();
        const uint64_t pol_q = l2_policy_evict_last();
        long long pos = 0;
        long long last_pos[kAttnStages] = {-1, -1, -1, -1};
        int p = 0;
        for (long long u = u_first; u <= u_last; ++u, ++p) {
            const int pb = p & 1;
            const long long lo = max(s_begin, u * K), hi = min(s_end, (u + 1) * K);
            const int b = static_cast<int>(u / d.Hkv), h = static_cast<int>(u % d.Hkv);
            if (lane == 0 && p >= 2) attn_wait(&bar[kBarLFree + pb], ((p >> 1) - 1) & 1, s_abort);
            __syncwarp();
            // the occupied slots of the piece, in slot order: (slot in unit) << 5 | valid tokens
            int* list = s_list + pb * kAttnMaxList;
            const int ctx = ctx_len[b];
            int n = 0;
            for (long long base = lo; base < hi; base += 32) {
                const long long s = base + lane;
                int nv = 0;
                if (s < hi) {
                    int blk = slot_table[s];
                    if (blk < -1 || blk >= d.N) {
                        raise_dev_error(OASIS_DEVERR_ID_RANGE);
                        blk = -1;
                    }
                    if (blk >= 0) nv = min(kBlockTokens, max(0, ctx - blk * kBlockTokens));
                }
                const unsigned m = __ballot_sync(0xFFFFFFFFu, nv > 0);
                if (nv > 0) list[n + __popc(m & ((1u << lane) - 1u))] = (static_cast<int>(s - u * K) << 5) | nv;
                n += __popc(m);
            }
            __syncwarp();
            if (lane == 0) {
                s_nlist[pb] = n;
                __threadfence_block();
                mbar_arrive(&bar[kBarLFull + pb]);
                // the unit's query rows: box {64 columns, G heads, Qn rows} per 64-column half
                if (p >= 2) attn_wait(&bar[kBarQFree + pb], ((p >> 1) - 1) & 1, s_abort);
                mbar_arrive_expect_tx(&bar[kBarQFull + pb], static_cast<uint32_t>(rows) * kRowBytes);
                if (!*s_abort) {
                    uint8_t* q_dst = sQ + pb * 2 * kAttnRegion;
                    tma_load_3d(q_dst, &tm_q, &bar[kBarQFull + pb], 0, h * G, b * d.Qn, pol_q);
                    tma_load_3d(q_dst + kAttnRegion, &tm_q, &bar[kBarQFull + pb], 64, h * G, b * d.Qn, pol_q);
                }
                const int ntiles = (n + kAttnTileSlots - 1) / kAttnTileSlots;
                for (int i = 0; i < ntiles; ++i, ++pos) {
                    const int stage = static_cast<int>(pos % kAttnStages);
                    if (pos >= kAttnStages)
                        attn_wait(&bar[kBarEmpty + stage], static_cast<uint32_t>((pos / kAttnStages - 1) & 1),
                                  s_abort);
                    const int ns = min(kAttnTileSlots, n - i * kAttnTileSlots);
                    mbar_arrive_expect_tx(&bar[kBarFull + stage], static_cast<uint32_t>(ns) * kBlockBytes);
                    last_pos[stage] = pos;
                    if (*s_abort) continue;
                    uint8_t* st = ring + stage * kAttnStageBytes;
                    for (int j = 0; j < ns; ++j) {
                        const int slot = list[i * kAttnTileSlots + j] >> 5;
                        const int y = static_cast<int>((u * K + slot) * (2 * kBlockTokens));
                        const int off = j * (kBlockTokens * 128);
                        tma_load_2d(st + 0 * kAttnRegion + off, &tm_pool, &bar[kBarFull + stage], 0, y, pol_kv);
                        tma_load_2d(st + 1 * kAttnRegion + off, &tm_pool, &bar[kBarFull + stage], 64, y, pol_kv);
                        tma_load_2d(st + 2 * kAttnRegion + off, &tm_pool, &bar[kBarFull + stage], 0,
                                    y + kBlockTokens, pol_kv);
                        tma_load_2d(st + 3 * kAttnRegion + off, &tm_pool, &bar[kBarFull + stage], 64,
                                    y + kBlockTokens, pol_kv);
                    }
                }
            }
            __syncwarp();
            n = __shfl_sync(0xFFFFFFFFu, n, 0);
            pos = __shfl_sync(0xFFFFFFFFu, pos, 0);
        }
        // no copy may still be writing this CTA's shared memory when it exits
        if (lane == 0)
            for (int s = 0; s < kAttnStages; ++s)
                if (last_pos[s] >= 0) mbar_wait(&bar[kBarFull + s], static_cast<uint32_t>((last_pos[s] / kAttnStages) & 1));
    } else if (warp == 1) {
        // =================================================== MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16_f32(kAttnRows, kAttnTileSlots * kBlockTokens);
            constexpr uint32_t idesc_pv = umma_idesc_bf16_f32_bmn(kAttnRows, kHeadDim);
            long long pos = 0;
            int p = 0;
            bool have_prev = false, prev_first = false, prev_last = false;
            long long prev_pos = 0;
            int prev_ns = 0;
            auto issue_pv = [&](long long ppos, int pns, bool pfirst, bool plast) {
                const int sb = static_cast<int>(ppos & 1);
                const int stage = static_cast<int>(ppos % kAttnStages);
                const bool ok = attn_wait(&bar[kBarPFull + sb], static_cast<uint32_t>((ppos >> 1) & 1), s_abort);
                tc_fence_after_sync();
                if (ok) {
                    const uint32_t pa = smem_addr(sP + sb * 2 * kAttnRegion);
                    const uint32_t va = smem_addr(ring + stage * kAttnStageBytes + 2 * kAttnRegion);
                    for (int kk = 0; kk < pns; ++kk) {
                        const uint64_t bd = umma_desc_sw128_lbo_sbo(va + kk * (kBlockTokens * 128), kAttnRegion, 1024);
                        umma_bf16(tmem_o, umma_desc_sw128_lbo_sbo(pa + kk * 32, 16, 1024), bd, idesc_pv,
                                  (pfirst && kk == 0) ? 0u : 1u);
                        umma_bf16(tmem_o, umma_desc_sw128_lbo_sbo(pa + kAttnRegion + kk * 32, 16, 1024), bd,
                                  idesc_pv, 1u);
                    }
                }
                umma_commit(&bar[kBarEmpty + stage]);
                umma_commit(&bar[kBarPFree + sb]);
                if (plast) umma_commit(&bar[kBarODone]);
            };
            for (long long u = u_first; u <= u_last; ++u, ++p) {
                const int pb = p & 1;
                attn_wait(&bar[kBarLFull + pb], static_cast<uint32_t>((p >> 1) & 1), s_abort);
                const int n = s_nlist[pb];
                const int ntiles = (n + kAttnTileSlots - 1) / kAttnTileSlots;
                attn_wait(&bar[kBarQFull + pb], static_cast<uint32_t>((p >> 1) & 1), s_abort);
                const uint32_t qa = smem_addr(sQ + pb * 2 * kAttnRegion);
                for (int i = 0; i < ntiles; ++i, ++pos) {
                    const int stage = static_cast<int>(pos % kAttnStages);
                    const int sb = static_cast<int>(pos & 1);
                    bool ok = attn_wait(&bar[kBarFull + stage], static_cast<uint32_t>((pos / kAttnStages) & 1),
                                        s_abort);
                    if (pos >= 2) ok = attn_wait(&bar[kBarSFree + sb], static_cast<uint32_t>(((pos >> 1) - 1) & 1),
                                                 s_abort) && ok;
                    tc_fence_after_sync();
                    if (ok) {
                        const uint32_t ka = smem_addr(ring + stage * kAttnStageBytes);
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks) {
                            const uint32_t off = (ks >> 2) * kAttnRegion + (ks & 3) * 32;
                            umma_bf16(tmem + sb * 64, umma_desc_sw128_lbo_sbo(qa + off, 16, 1024),
                                      umma_desc_sw128_lbo_sbo(ka + off, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
                        }
                    }
                    umma_commit(&bar[kBarSFull + sb]);
                    if (have_prev) issue_pv(prev_pos, prev_ns, prev_first, prev_last);
                    have_prev = true;
                    prev_pos = pos;
                    prev_ns = min(kAttnTileSlots, n - i * kAttnTileSlots);
                    prev_first = i == 0;
                    prev_last = i == ntiles - 1;
                }
                umma_commit(&bar[kBarQFree + pb]);            // after the piece's last S
                mbar_arrive(&bar[kBarLFree + pb]);
            }
            if (have_prev) issue_pv(prev_pos, prev_ns, prev_first, prev_last);
            umma_commit(&bar[kBarFinal]);
            mbar_wait(&bar[kBarFinal], 0);
        }
        __syncwarp();
    } else {
        // ============================================ softmax / epilogue
        const int qd = warp & 3;                              // TMEM lane quadrant
        const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
        const int rA = 16 * qd + (lane >> 2), rB = rA + 8;   // this thread's query rows
        const bool realA = rA < rows, realB = rB < rows;
        const int cp = 2 * (lane & 3);                        // column pair within each 8-column chunk
        long long pos = 0;
        int nonempty = 0;
        int p = 0;
        for (long long u = u_first; u <= u_last; ++u, ++p) {
            const int pb = p & 1;
            attn_wait(&bar[kBarLFull + pb], static_cast<uint32_t>((p >> 1) & 1), s_abort);
            const int n = s_nlist[pb];
            const int* list = s_list + pb * kAttnMaxList;
            const int ntiles = (n + kAttnTileSlots - 1) / kAttnTileSlots;
            float mA = kNegInf, mB = kNegInf, lA = 0.f, lB = 0.f;
            for (int i = 0; i < ntiles; ++i, ++pos) {
                const int sb = static_cast<int>(pos & 1);
                const int stage = static_cast<int>(pos % kAttnStages);
                const int ns = min(kAttnTileSlots, n - i * kAttnTileSlots);
                int nvj[kAttnTileSlots];
#pragma unroll
                for (int j = 0; j < kAttnTileSlots; ++j) nvj[j] = j < ns ? (list[i * kAttnTileSlots + j] & 31) : 0;
                attn_wait(&bar[kBarSFull + sb], static_cast<uint32_t>((pos >> 1) & 1), s_abort);
                tc_fence_after_sync();
                uint32_t v[32];
                tmem_ld_16x256b_x8(tmem + lane_base + sb * 64, v);
                tmem_ld_wait();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar[kBarSFree + sb]);
                float s[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int j = c >> 1;                      // slot of this chunk
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int tt = (c & 1) * 8 + cp + e;   // token within the slot
                        const bool ok = tt < nvj[j];
                        s[4 * c + e] = ok ? __uint_as_float(v[4 * c + e]) : kNegInf;
                        s[4 * c + 2 + e] = ok ? __uint_as_float(v[4 * c + 2 + e]) : kNegInf;
                    }
                }
                float mxA = kNegInf, mxB = kNegInf;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    mxA = fmaxf(mxA, fmaxf(s[4 * c], s[4 * c + 1]));
                    mxB = fmaxf(mxB, fmaxf(s[4 * c + 2], s[4 * c + 3]));
                }
                mxA = fmaxf(mxA, __shfl_xor_sync(0xFFFFFFFFu, mxA, 1));
                mxA = fmaxf(mxA, __shfl_xor_sync(0xFFFFFFFFu, mxA, 2));
                mxB = fmaxf(mxB, __shfl_xor_sync(0xFFFFFFFFu, mxB, 1));
                mxB = fmaxf(mxB, __shfl_xor_sync(0xFFFFFFFFu, mxB, 2));
                mxA *= scale_log2;
                mxB *= scale_log2;
                // P buffer sb is free once PV of tile pos-2 has completed
                if (pos >= 2) attn_wait(&bar[kBarPFree + sb], static_cast<uint32_t>(((pos >> 1) - 1) & 1), s_abort);
                // running max: moved only by more than 2^8 (exact lse for any reference)
                float alA = 1.f, alB = 1.f;
                bool resc = false;
                if (mxA > mA + 8.f) {
                    if (i > 0) {
                        alA = exp2f(mA - mxA);
                        resc = true;
                    }
                    mA = mxA;
                }
                if (mxB > mB + 8.f) {
                    if (i > 0) {
                        alB = exp2f(mB - mxB);
                        resc = true;
                    }
                    mB = mxB;
                }
                lA *= alA;
                lB *= alB;
                if (__any_sync(0xFFFFFFFFu, resc)) {
                    // PV of tile pos-1 must have landed in O before it is rescaled
                    attn_wait(&bar[kBarPFree + (sb ^ 1)], static_cast<uint32_t>(((pos - 1) >> 1) & 1), s_abort);
                    tc_fence_after_sync();
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t o[32];
                        tmem_ld_16x256b_x8(tmem_o + lane_base + half * 64, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            o[4 * c + 0] = __float_as_uint(__uint_as_float(o[4 * c + 0]) * alA);
                            o[4 * c + 1] = __float_as_uint(__uint_as_float(o[4 * c + 1]) * alA);
                            o[4 * c + 2] = __float_as_uint(__uint_as_float(o[4 * c + 2]) * alB);
                            o[4 * c + 3] = __float_as_uint(__uint_as_float(o[4 * c + 3]) * alB);
                        }
                        tmem_st_16x256b_x8(tmem_o + lane_base + half * 64, o);
                    }
                    tmem_st_wait();
                }
                // probabilities: head + remainder in bf16, written 128-byte swizzled
                uint8_t* p_head = sP + sb * 2 * kAttnRegion;
                uint8_t* p_rest = p_head + kAttnRegion;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float a0 = exp2f(fmaf(s[4 * c + 0], scale_log2, -mA));
                    const float a1 = exp2f(fmaf(s[4 * c + 1], scale_log2, -mA));
                    const float b0 = exp2f(fmaf(s[4 * c + 2], scale_log2, -mB));
                    const float b1 = exp2f(fmaf(s[4 * c + 3], scale_log2, -mB));
                    lA += a0 + a1;
                    lB += b0 + b1;
                    if (realA) {
                        const uint32_t hd = pack_bf16x2(a0, a1);
                        const uint32_t rs = pack_bf16x2(a0 - bf16_lo(hd), a1 - bf16_hi(hd));
                        const int off = rA * 128 + ((c ^ (rA & 7)) << 4) + cp * 2;
                        *reinterpret_cast<uint32_t*>(p_head + off) = hd;
                        *reinterpret_cast<uint32_t*>(p_rest + off) = rs;
                    }
                    if (realB) {
                        const uint32_t hd = pack_bf16x2(b0, b1);
                        const uint32_t rs = pack_bf16x2(b0 - bf16_lo(hd), b1 - bf16_hi(hd));
                        const int off = rB * 128 + ((c ^ (rB & 7)) << 4) + cp * 2;
                        *reinterpret_cast<uint32_t*>(p_head + off) = hd;
                        *reinterpret_cast<uint32_t*>(p_rest + off) = rs;
                    }
                }
                // value rows past the context of a partly filled block read as zero
                // (their weights are zero, and zero times a non-finite stale value is not)
                if (qd < ns && nvj[qd] < kBlockTokens) {
                    // the tile's copy is complete (already awaited by the MMA thread; this
                    // wait returns at once and orders the copy before these writes)
                    attn_wait(&bar[kBarFull + stage], static_cast<uint32_t>((pos / kAttnStages) & 1), s_abort);
                    uint8_t* vbase = ring + stage * kAttnStageBytes + 2 * kAttnRegion + qd * (kBlockTokens * 128);
                    const int first_row = nvj[qd];
                    for (int k = lane; k < (kBlockTokens - first_row) * 16; k += 32) {
                        const int row = first_row + (k >> 4), chunk = k & 15;
                        *reinterpret_cast<uint4*>(vbase + (chunk >> 3) * kAttnRegion + row * 128 + (chunk & 7) * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar[kBarPFull + sb]);
            }

            // ------------------------------------------------- epilogue
            if (ntiles > 0) {
                attn_wait(&bar[kBarODone], static_cast<uint32_t>(nonempty & 1), s_abort);
                ++nonempty;
                tc_fence_after_sync();
            }
            lA += __shfl_xor_sync(0xFFFFFFFFu, lA, 1);
            lA += __shfl_xor_sync(0xFFFFFFFFu, lA, 2);
            lB += __shfl_xor_sync(0xFFFFFFFFu, lB, 1);
            lB += __shfl_xor_sync(0xFFFFFFFFu, lB, 2);
            const float invA = lA > 0.f ? 1.f / lA : 0.f, invB = lB > 0.f ? 1.f / lB : 0.f;
            const bool direct = u * K >= s_begin && (u + 1) * K <= s_end;
            const int b = static_cast<int>(u / d.Hkv), h = static_cast<int>(u % d.Hkv);
            const long long pidx = gs + u;                    // this CTA's partial of unit u
            const long long orowA = (static_cast<long long>(b) * d.Qn + rA / G) * d.Hq + h * G + rA % G;
            const long long orowB = (static_cast<long long>(b) * d.Qn + rB / G) * d.Hq + h * G + rB % G;
            float* dstA = direct ? out + orowA * kHeadDim : ws_o + (pidx * rows + rA) * kHeadDim;
            float* dstB = direct ? out + orowB * kHeadDim : ws_o + (pidx * rows + rB) * kHeadDim;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t o[32];
                if (ntiles > 0) {
                    tmem_ld_16x256b_x8(tmem_o + lane_base + half * 64, o);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int k = 0; k < 32; ++k) o[k] = 0u;
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int col = half * 64 + 8 * c + cp;
                    if (realA)
                        *reinterpret_cast<float2*>(dstA + col) =
                            make_float2(__uint_as_float(o[4 * c]) * invA, __uint_as_float(o[4 * c + 1]) * invA);
                    if (realB)
                        *reinterpret_cast<float2*>(dstB + col) = make_float2(__uint_as_float(o[4 * c + 2]) * invB,
                                                                             __uint_as_float(o[4 * c + 3]) * invB);
                }
            }
            tc_fence_before_sync();
            if ((lane & 3) == 0) {
                const float l2A = lA > 0.f ? mA + log2f(lA) : kNegInf;
                const float l2B = lB > 0.f ? mB + log2f(lB) : kNegInf;
                if (direct) {
                    if (realA) lse_out[orowA] = lA > 0.f ? l2A * kLn2 : kNegInf;
                    if (realB) lse_out[orowB] = lB > 0.f ? l2B * kLn2 : kNegInf;
                } else {
                    if (realA) ws_lse[pidx * rows + rA] = l2A;
                    if (realB) ws_lse[pidx * rows + rB] = l2B;
                }
            }
            if (!direct) {
                __threadfence();
                named_bar_sync(1, 128);
                if (warp == 2 && lane == 0) {
                    long long first, last;
                    attn_unit_streams(u, K, n_streams, T, &first, &last);
                    const int old = atomicAdd(ws_ticket + u, 1);
                    *s_last = old == static_cast<int>(last - first) ? 1 : 0;
                }
                named_bar_sync(1, 128);
                if (*s_last) {
                    __threadfence();
                    long long first, last;
                    attn_unit_streams(u, K, n_streams, T, &first, &last);
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const int r = rr == 0 ? rA : rB;
                        if (r >= rows) continue;
                        const long long orow = rr == 0 ? orowA : orowB;
                        float M = kNegInf;
                        for (long long sp = first; sp <= last; ++sp) M = fmaxf(M, __ldcg(ws_lse + (sp + u) * rows + r));
                        float L = 0.f;
                        float2 acc[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k) acc[k] = make_float2(0.f, 0.f);
                        if (M != kNegInf) {
                            for (long long sp = first; sp <= last; ++sp) {
                                const float lj = __ldcg(ws_lse + (sp + u) * rows + r);
                                if (lj == kNegInf) continue;             // empty partial: its output is not read
                                const float w = exp2f(lj - M);
                                L += w;
                                const float* src = ws_o + ((sp + u) * rows + r) * kHeadDim;
#pragma unroll
                                for (int k = 0; k < 16; ++k) {
                                    const int col = (k >> 3) * 64 + 8 * (k & 7) + cp;
                                    const float2 x = __ldcg(reinterpret_cast<const float2*>(src + col));
                                    acc[k].x += w * x.x;
                                    acc[k].y += w * x.y;
                                }
                            }
                        }
                        const float inv = L > 0.f ? 1.f / L : 0.f;
                        float* dst = out + orow * kHeadDim;
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const int col = (k >> 3) * 64 + 8 * (k & 7) + cp;
                            *reinterpret_cast<float2*>(dst + col) = make_float2(acc[k].x * inv, acc[k].y * inv);
                        }
                        if ((lane & 3) == 0) lse_out[orow] = L > 0.f ? (M + log2f(L)) * kLn2 : kNegInf;
                    }
                    if (warp == 2 && lane == 0) ws_ticket[u] = 0;         // ready for the next call
                }
            }
            named_bar_sync(1, 128);                                         // every warp is done with the list
            if (warp == 2 && lane == 0) {
                *s_last = 0;
                mbar_arrive(&bar[kBarLFree + pb]);
            }
        }
    }

    // ---------------------------------------------------------- teardown
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc(tmem, kAttnTmemCols);
}

}  // namespace oasis
