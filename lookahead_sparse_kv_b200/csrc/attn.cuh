// attn.cuh - sparse GQA decode attention over the resident pool slots, on
// the 5th-generation tensor cores.
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching, Figure 7 (right): the verification query and the drafts are
// attended in one pass over the resident sparse working set; Figure 9: the
// per-head slot table says which block each pool slot holds.
//
// Shapes.  A (sequence, KV head) "unit" has rows = Qn*G query rows (at most
// 64) and K pool slots of 16 tokens.  Decode has few query rows and many
// tokens, so the tokens are the MMA's M dimension:
//   S^T [128 tokens x NR]   = K_tile [128 x 128] . Q^T        8 MMAs, both K-major
//   O^T [128 dims x 2 NR]  += V_tile^T . [P_head | P_rest]^T [128 tokens x 2 NR]
//                             one MMA per occupied slot (16 tokens), both
//                             operands MN-major: V is read in place, P^T is
//                             written one row per token as a bf16 head and a
//                             bf16 remainder (~16 significant bits), side by
//                             side along N, so head and remainder products land
//                             in two column ranges that the epilogue adds; with
//                             32 rows the two share a 128-B row, with 64 they
//                             take a region each; P^T is double-buffered, so a
//                             tile's softmax overlaps the previous tile's product
// NR = 32 or 64 is the row count padded to the MMA's N.  A tile is 8 pool
// slots (128 tokens).  In TMEM, lane i of S^T is token i of the tile (a
// softmax thread owns a token and reads its NR scores), lane i of O^T is
// head-dimension channel i (an epilogue thread owns a channel and writes it
// for every row), so only real rows are ever exponentiated and every TMEM
// access is a plain 32x32b row per thread.
//
// Work split.  A unit's slots are cut into chunks of `ct` tiles (`cpu`
// chunks per unit, `nc` in all).  Persistent CTAs (at most one per SM) take
// chunks from an atomic counter in the workspace, so a CTA that runs slowly
// (beside a gather on its SM, say) simply takes fewer.  A chunk that is a
// whole unit is normalised and written directly; otherwise it writes a
// normalised partial (output, log2-sum-exp) and takes a ticket, and the last
// chunk of the unit to finish merges the unit's partials (still in L2) and
// resets the ticket.  The last CTA to exit resets the chunk counter, so the
// workspace is ready for the next call.
//
// Roles (16 warps, mbarriers for every hand-off, every wait bounded):
//   warp 15    lister: takes chunks (the next one is requested while the
//              current one is listed), lists a chunk's tiles that hold a
//              valid token (valid-token count of each slot) and loads the
//              unit's query rows;
//   warp 12    loader: lane 0 streams the listed tiles' K, lane 1 their V,
//              through two 2-stage TMA rings (per tile and tensor two 16-KiB boxes of 8 slots x
//              16 rows x 64 columns, 128-byte swizzle).
//   warp 13    issues S^T (and holds the TMEM allocation).
//   warp 14    issues O^T; a free slot's product is not issued.
//   warps 0-7  softmax, one token and half the rows per thread (two warps per
//              TMEM lane quadrant).  A chunk's running max of a
//              row starts at the score of the chunk's first valid token and
//              moves only when a tile exceeds it by more than 2^32 (found with
//              one barrier-wide vote per tile; probabilities stay below 2^32,
//              far inside fp32 and bf16 range, and any m gives the exact
//              log-sum-exp); then the tile's row maxima are reduced across
//              the four warps and O^T and the row sums are rescaled.  Value rows past the context in a partly
//              filled slot are zeroed so stale bytes never meet a zero
//              weight.
//   warps 8-11 epilogue, one channel per thread, double-buffered against
//              the next chunk (two O^T accumulators in TMEM).
#pragma once

#include "common.cuh"

namespace oasis {

constexpr int kAttnTileSlots = 8;                                  // slots per tile
constexpr int kAttnTileTokens = kAttnTileSlots * kBlockTokens;     // 128: the MMA's M
constexpr int kAttnHalf = kAttnTileTokens * 128;                   // one 64-column half of a tile: 16 KiB
constexpr int kAttnStageBytes = 2 * kAttnHalf;                     // K (or V) of one tile
constexpr int kAttnQHalf = 64 * 128;                               // 64 query rows x 128 B
constexpr int kAttnMaxChunkTiles = 16;
constexpr int kAttnInfoInts = 8 + 4 * kAttnMaxChunkTiles;          // chunk header + 4 ints per tile
constexpr int kAttnSoftmaxWarps = 8;                              // warps 0-7 (two per TMEM quadrant)
constexpr int kAttnEpiWarp = 8;                                    // warps 8-11
constexpr int kAttnLoaderWarp = 12, kAttnSWarp = 13, kAttnOWarp = 14, kAttnListerWarp = 15;
constexpr int kAttnThreads = 32 * 16;
constexpr int kAttnTmemCols = 512;                                 // S^T x 2 (64 columns each), O^T x 2 (2 NR each), row sums
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kAttnLazy = 32.f;                                  // rescale when a score passes m + 32 (log2)

// shared memory, from the 1024-B aligned base: the K and V rings, the small
// arrays, then the query rows and P^T, whose size depends on the row count
constexpr int kAttnOffK = 0;                                       // K ring, 2 stages
constexpr int kAttnOffV = kAttnOffK + 2 * kAttnStageBytes;         // V ring, 2 stages
constexpr int kAttnOffInfo = kAttnOffV + 2 * kAttnStageBytes;      // 2 chunk descriptions
constexpr int kAttnOffBar = kAttnOffInfo + 2 * kAttnInfoInts * 4;
constexpr int kAttnNumBars = 32;
constexpr int kAttnOffMisc = kAttnOffBar + kAttnNumBars * 8;       // 8 ints
constexpr int kAttnOffM = kAttnOffMisc + 32;                       // [2][64] running max (log2 units)
constexpr int kAttnOffAlpha = kAttnOffM + 2 * 64 * 4;              // [64] rescale factors of a tile
constexpr int kAttnOffWmax = kAttnOffAlpha + 64 * 4;               // [4][64] per-warp tile maxima
constexpr int kAttnOffLw = kAttnOffWmax + 4 * 64 * 4;              // [2][4][64] per-warp row sums
constexpr int kAttnOffFin = kAttnOffLw + 2 * 4 * 64 * 4;           // [2][64] 1/sum, [2][64] log2-sum-exp
constexpr int kAttnMaxChunks = 8;                                  // chunks per unit (merge weights)
constexpr int kAttnOffMw = kAttnOffFin + 4 * 64 * 4;               // [64][8] merge weights
constexpr int kAttnOffThr = kAttnOffMw + 64 * kAttnMaxChunks * 4;  // [2][64] raw-score thresholds
constexpr int kAttnOffQ = (kAttnOffThr + 2 * 64 * 4 + 1023) / 1024 * 1024;
// Query buffers (2 halves each) and P^T buffers.  With 32 rows a 128-B row
// per token holds P^T's head (bytes 0-63 of the row before swizzling) and
// remainder (64-127), and the query rows are double-buffered across chunks;
// with 64 rows head and remainder fill a [128 tokens][128 B] region each, and
// a single query buffer leaves room for the second P^T buffer.
constexpr int attn_q_bufs(int nr) { return nr == 64 ? 1 : 2; }
constexpr int attn_p_buf_bytes(int nr) { return (nr == 64 ? 2 : 1) * kAttnHalf; }
constexpr int attn_off_p(int nr) { return kAttnOffQ + attn_q_bufs(nr) * 2 * kAttnQHalf; }
constexpr int attn_smem(int nr) { return attn_off_p(nr) + 2 * attn_p_buf_bytes(nr) + 1024; }   // + alignment slack
static_assert(attn_smem(32) <= 227 * 1024 && attn_smem(64) <= 227 * 1024, "attention shared memory");

// mbarriers ([2] = one per ring stage / buffer)
constexpr int kBarKFull = 0;     // K tile landed (producer expect_tx)
constexpr int kBarKEmpty = 2;    // K tile read by S^T (commit)
constexpr int kBarVFull = 4;     // V tile landed
constexpr int kBarVEmpty = 6;    // V tile read by O^T (commit)
constexpr int kBarSFull = 8;     // S^T computed (commit)
constexpr int kBarSFree = 10;    // S^T read by the 4 softmax warps
constexpr int kBarPFull = 12;    // P^T written by the 4 softmax warps (per P^T buffer)
constexpr int kBarPFree = 14;    // P^T read by O^T (commit)
constexpr int kBarQFull = 16;    // chunk's query rows landed
constexpr int kBarQFree = 18;    // query rows no longer read (commit after the chunk's last S^T)
constexpr int kBarLFull = 20;    // chunk description written (producer)
constexpr int kBarLFree = 22;    // description read by every consumer (kAttnLFreeCount arrivals)
constexpr int kBarODone = 24;    // chunk's last O^T product completed (commit)
constexpr int kBarOFree = 26;    // O^T accumulator, running max and row sums read by the epilogue
constexpr int kBarSMDone = 28;   // chunk's row sums written by the 4 softmax warps
constexpr int kBarFinalS = 30;   // teardown: every S^T issued has completed
constexpr int kBarFinalO = 31;   // teardown: every O^T issued has completed
constexpr int kAttnLFreeCount = 16;   // 14 consumer warps + the loader's K and V lanes

// named barriers (0 is __syncthreads); the softmax warps of the low rows (warps
// 0-3) and of the high rows (warps 4-7) each have their own pair
constexpr uint32_t kNbSoftmax = 1, kNbSoftmaxVote = 2, kNbEpi = 3, kNbEpiVote = 4;
constexpr uint32_t kNbSoftmaxHi = 5, kNbSoftmaxVoteHi = 6;

// Chunking of the attention work (host and device agree through these).
struct AttnChunks {
    int ct;    // tiles per chunk
    int cpu;   // chunks per unit
    int nc;    // chunks in all
};

// 2^x on the multi-function unit (approximate, |rel err| about 2^-22; -inf -> +0).
__device__ __forceinline__ float attn_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Butterfly reduce-scatter over the warp: v[0..31] in every lane; on return
// lane t holds the max (or the sum) over all lanes of v[t].  v is clobbered.
template <bool kMax>
__device__ __forceinline__ float warp_reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
        const bool up = (lane & w) != 0;
#pragma unroll
        for (int k = 0; k < w; ++k) {
            const float send = up ? v[k] : v[k + w];
            const float keep = up ? v[k + w] : v[k];
            const float got = __shfl_xor_sync(0xFFFFFFFFu, send, w);
            v[k] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
    return v[0];
}

// The same over 16 values: the two half-warps are folded first, then lane t
// (and t + 16) holds the result for v[t & 15].
template <bool kMax>
__device__ __forceinline__ float warp_reduce_scatter16(float (&v)[16], int lane) {
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float got = __shfl_xor_sync(0xFFFFFFFFu, v[k], 16);
        v[k] = kMax ? fmaxf(v[k], got) : v[k] + got;
    }
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1) {
        const bool up = (lane & w) != 0;
#pragma unroll
        for (int k = 0; k < w; ++k) {
            const float send = up ? v[k] : v[k + w];
            const float keep = up ? v[k + w] : v[k];
            const float got = __shfl_xor_sync(0xFFFFFFFFu, send, w);
            v[k] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
    return v[0];
}

template <int NR>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_q, Dims d, const int32_t* __restrict__ slot_table,
                       const int32_t* __restrict__ ctx_len, float scale_log2, AttnChunks ch,
                       float* __restrict__ out, float* __restrict__ lse_out, float* ws_o, float* ws_lse,
                       int* ws_ticket, int* ws_sched) {
    static_assert(NR == 32 || NR == 64, "rows are padded to 32 or 64");
    constexpr int kPBufs = 2;                                     // P^T buffers
    constexpr int kPBufBytes = attn_p_buf_bytes(NR);
    constexpr int kQBufs = attn_q_bufs(NR);                      // query-row buffers
    // TMEM columns: S^T buffers at 0 and 64, O^T buffers (head and remainder
    // products side by side) at 128 and 128 + 2 NR, 64-row sums after them
    constexpr uint32_t kOCol = 128, kOStride = 2 * NR;
    const float kNegInf = -__int_as_float(0x7f800000);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem + kAttnOffK;
    uint8_t* sV = smem + kAttnOffV;
    uint8_t* sQ = smem + kAttnOffQ;
    uint8_t* sP = smem + attn_off_p(NR);
    int* s_info = reinterpret_cast<int*>(smem + kAttnOffInfo);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kAttnOffBar);
    int* misc = reinterpret_cast<int*>(smem + kAttnOffMisc);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(misc);
    volatile int* s_abort = misc + 1;
    volatile int* s_last = misc + 2;
    float* s_m = reinterpret_cast<float*>(smem + kAttnOffM);
    float* s_alpha = reinterpret_cast<float*>(smem + kAttnOffAlpha);
    float* s_wmax = reinterpret_cast<float*>(smem + kAttnOffWmax);
    float* s_lw = reinterpret_cast<float*>(smem + kAttnOffLw);
    float* s_fin = reinterpret_cast<float*>(smem + kAttnOffFin);
    float* s_mw = reinterpret_cast<float*>(smem + kAttnOffMw);
    float* s_thr = reinterpret_cast<float*>(smem + kAttnOffThr);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = d.K;
    const int G = d.G();
    const int rows = d.Qn * G;

    // ---------------------------------------------------------- set-up
    if (tid == 0) {
        for (int i = 0; i < kAttnNumBars; ++i) {
            int cnt = 1;
            if (i == kBarSFree || i == kBarSFree + 1 || i == kBarPFull || i == kBarPFull + 1 || i == kBarSMDone ||
                i == kBarSMDone + 1)
                cnt = kAttnSoftmaxWarps;
            if (i == kBarLFree || i == kBarLFree + 1) cnt = kAttnLFreeCount;
            mbar_init(&bar[i], cnt);
        }
        fence_mbar_init();
        *s_abort = 0;
        *s_last = 0;
    }
    if (warp == kAttnSWarp) {
        tmem_alloc(s_tmem, kAttnTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *s_tmem;

    if (warp == kAttnListerWarp) {
        // ======================================================= lister
        if (lane == 0) prefetch_tensormap(&tm_q);
        const uint64_t pol_q = l2_policy_evict_last();
        // the first chunk of each CTA is its block index (grid <= chunks), the
        // rest come from the counter, numbered from the grid size on
        int c_next = static_cast<int>(blockIdx.x);
        for (int p = 0;; ++p) {
            const int pb = p & 1;
            int* info = s_info + pb * kAttnInfoInts;
            if (lane == 0 && p >= 2) cta_wait(&bar[kBarLFree + pb], ((p >> 1) - 1) & 1, s_abort);
            int c = c_next;
            if (lane == 0 && *s_abort) c = ch.nc;
            c = __shfl_sync(0xFFFFFFFFu, c, 0);
            if (c >= ch.nc) {
                if (lane == 0) {
                    info[0] = -1;
                    mbar_arrive(&bar[kBarLFull + pb]);
                }
                break;
            }
            if (lane == 0) c_next = static_cast<int>(gridDim.x) + atomicAdd(ws_sched, 1);   // lands while this chunk is listed
            const int u = c / ch.cpu, j = c - u * ch.cpu;
            const int lo = j * ch.ct * kAttnTileSlots, hi = min(lo + ch.ct * kAttnTileSlots, K);
            const int b = u / d.Hkv, h = u - b * d.Hkv;
            const int ctx = ctx_len[b];
            const int ntiles = (hi - lo + kAttnTileSlots - 1) / kAttnTileSlots;   // <= 16
            // lane i lists tile i: valid-token count of each of its 8 slots, a byte each
            uint32_t nvlo = 0u, nvhi = 0u;
            bool any = false;
            if (lane < ntiles) {
                const int s0 = lo + kAttnTileSlots * lane;
                int blk[kAttnTileSlots];
#pragma unroll
                for (int jj = 0; jj < kAttnTileSlots; ++jj)
                    blk[jj] = s0 + jj < hi ? slot_table[static_cast<long long>(u) * K + s0 + jj] : -1;
#pragma unroll
                for (int jj = 0; jj < kAttnTileSlots; ++jj) {
                    int bk = blk[jj];
                    if (bk < -1 || bk >= d.N) {
                        raise_dev_error(OASIS_DEVERR_ID_RANGE);
                        bk = -1;
                    }
                    const int nv = bk >= 0 ? min(kBlockTokens, max(0, ctx - bk * kBlockTokens)) : 0;
                    if (jj < 4)
                        nvlo |= static_cast<uint32_t>(nv) << (8 * jj);
                    else
                        nvhi |= static_cast<uint32_t>(nv) << (8 * (jj - 4));
                    any |= nv > 0;
                }
            }
            const unsigned m = __ballot_sync(0xFFFFFFFFu, any);
            const int n = __popc(m);
            if (any) {
                int* e = info + 8 + 4 * __popc(m & ((1u << lane) - 1u));
                e[0] = lo + kAttnTileSlots * lane;
                e[1] = static_cast<int>(nvlo);
                e[2] = static_cast<int>(nvhi);
            }
            __syncwarp();
            if (lane == 0) {
                info[0] = n;
                info[1] = c;
                info[2] = u;
                info[3] = ch.cpu;
                mbar_arrive(&bar[kBarLFull + pb]);
                // the unit's query rows: box {64 columns, G heads, Qn rows} per 64-column half
                // (after the S^T products of the chunk that last used the buffer)
                if (p >= kQBufs) cta_wait(&bar[kBarQFree + ((p - kQBufs) & 1)], ((p - kQBufs) >> 1) & 1, s_abort);
                mbar_arrive_expect_tx(&bar[kBarQFull + pb], static_cast<uint32_t>(rows) * kRowBytes);
                if (!*s_abort) {
                    uint8_t* q_dst = sQ + (p % kQBufs) * 2 * kAttnQHalf;
                    tma_load_3d(q_dst, &tm_q, &bar[kBarQFull + pb], 0, h * G, b * d.Qn, pol_q);
                    tma_load_3d(q_dst + kAttnQHalf, &tm_q, &bar[kBarQFull + pb], 64, h * G, b * d.Qn, pol_q);
                }
            }
            __syncwarp();
        }
    } else if (warp == kAttnLoaderWarp) {
        // ======================================================= loader
        // lane 0 streams K, lane 1 streams V, each through its own 2-stage
        // ring: a K tile is requested as soon as its stage's S^T product is
        // done, without waiting behind the V stage, which stays held until
        // the O^T product of its tile (after that tile's softmax)
        if (lane < 2) {
            const bool is_k = lane == 0;
            const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
            uint8_t* ring = is_k ? sK : sV;
            const int bar_full = is_k ? kBarKFull : kBarVFull, bar_empty = is_k ? kBarKEmpty : kBarVEmpty;
            prefetch_tensormap(tm);
            const uint64_t pol_kv = l2_policy_evict_first();
            int pos = 0;
            int last[2] = {-1, -1};
            for (int p = 0;; ++p) {
                const int pb = p & 1;
                if (!cta_wait(&bar[kBarLFull + pb], (p >> 1) & 1, s_abort)) break;
                const int* info = s_info + pb * kAttnInfoInts;
                const int n = info[0];
                if (n < 0) break;
                const int zu = info[2] * K;
                for (int i = 0; i < n; ++i, ++pos) {
                    const int st = pos & 1;
                    const int z = zu + info[8 + 4 * i];              // first pool slot of the tile
                    if (pos >= 2) cta_wait(&bar[bar_empty + st], ((pos >> 1) - 1) & 1, s_abort);
                    mbar_arrive_expect_tx(&bar[bar_full + st], kAttnStageBytes);
                    if (!*s_abort) {
                        last[st] = pos;
                        uint8_t* dst = ring + st * kAttnStageBytes;
                        tma_load_3d(dst, tm, &bar[bar_full + st], 0, 0, z, pol_kv);
                        tma_load_3d(dst + kAttnHalf, tm, &bar[bar_full + st], 64, 0, z, pol_kv);
                    }
                }
                mbar_arrive(&bar[kBarLFree + pb]);
            }
            // no copy may still be writing this CTA's shared memory when it exits
            for (int st = 0; st < 2; ++st)
                if (last[st] >= 0) mbar_wait(&bar[bar_full + st], static_cast<uint32_t>((last[st] >> 1) & 1));
        }
        __syncwarp();
    } else if (warp == kAttnSWarp) {
        // =========================================== S^T = K . Q^T issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16_f32(kAttnTileTokens, NR);
            int sp = 0;
            for (int p = 0;; ++p) {
                const int pb = p & 1;
                if (!cta_wait(&bar[kBarLFull + pb], (p >> 1) & 1, s_abort)) break;
                const int n = s_info[pb * kAttnInfoInts];
                if (n < 0) break;
                cta_wait(&bar[kBarQFull + pb], (p >> 1) & 1, s_abort);
                const uint32_t qa = smem_addr(sQ + (p % kQBufs) * 2 * kAttnQHalf);
                for (int i = 0; i < n; ++i, ++sp) {
                    const int st = sp & 1;
                    bool ok = cta_wait(&bar[kBarKFull + st], (sp >> 1) & 1, s_abort);
                    if (sp >= 2) ok = cta_wait(&bar[kBarSFree + st], ((sp >> 1) - 1) & 1, s_abort) && ok;
                    tc_fence_after_sync();
                    if (ok) {
                        const uint32_t ka = smem_addr(sK + st * kAttnStageBytes);
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks)
                            umma_bf16(tmem + st * 64,
                                      umma_desc_sw128_lbo_sbo(ka + (ks >> 2) * kAttnHalf + (ks & 3) * 32, 16, 1024),
                                      umma_desc_sw128_lbo_sbo(qa + (ks >> 2) * kAttnQHalf + (ks & 3) * 32, 16, 1024),
                                      idesc, ks > 0 ? 1u : 0u);
                    }
                    umma_commit(&bar[kBarKEmpty + st]);
                    umma_commit(&bar[kBarSFull + st]);
                }
                umma_commit(&bar[kBarQFree + pb]);                // after the chunk's last S^T
                mbar_arrive(&bar[kBarLFree + pb]);
            }
            umma_commit(&bar[kBarFinalS]);
            mbar_wait(&bar[kBarFinalS], 0);
        }
        __syncwarp();
    } else if (warp == kAttnOWarp) {
        // ======================================== O^T += V^T . P^T issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16_f32_amn_bmn(kHeadDim, 2 * NR);
            int pv = 0;
            for (int p = 0;; ++p) {
                const int pb = p & 1;
                if (!cta_wait(&bar[kBarLFull + pb], (p >> 1) & 1, s_abort)) break;
                const int* info = s_info + pb * kAttnInfoInts;
                const int n = info[0];
                if (n < 0) break;
                if (p >= 2) cta_wait(&bar[kBarOFree + pb], ((p >> 1) - 1) & 1, s_abort);
                const uint32_t d_o = tmem + kOCol + pb * kOStride;
                bool fresh = true;                                // the chunk's first product overwrites O^T
                for (int i = 0; i < n; ++i, ++pv) {
                    const int st = pv & 1;
                    const int pbuf = pv % kPBufs;
                    bool ok = cta_wait(&bar[kBarPFull + pbuf], (pv / kPBufs) & 1, s_abort);
                    ok = cta_wait(&bar[kBarVFull + st], (pv >> 1) & 1, s_abort) && ok;
                    tc_fence_after_sync();
                    if (ok) {
                        const uint32_t nvlo = static_cast<uint32_t>(info[8 + 4 * i + 1]);
                        const uint32_t nvhi = static_cast<uint32_t>(info[8 + 4 * i + 2]);
                        const uint32_t va = smem_addr(sV + st * kAttnStageBytes);
                        const uint32_t pa = smem_addr(sP + pbuf * kPBufBytes);
#pragma unroll
                        for (int kk = 0; kk < kAttnTileSlots; ++kk) {
                            const uint32_t nv = ((kk < 4 ? nvlo : nvhi) >> (8 * (kk & 3))) & 0xFFu;
                            if (nv == 0) continue;                // free slot: no product
                            const uint32_t off = kk * kBlockTokens * 128;
                            umma_bf16(d_o, umma_desc_sw128_lbo_sbo(va + off, kAttnHalf, 1024),
                                      umma_desc_sw128_lbo_sbo(pa + off, kAttnHalf, 1024), idesc, fresh ? 0u : 1u);
                            fresh = false;
                        }
                    }
                    umma_commit(&bar[kBarVEmpty + st]);
                    umma_commit(&bar[kBarPFree + pbuf]);
                }
                umma_commit(&bar[kBarODone + pb]);
                mbar_arrive(&bar[kBarLFree + pb]);
            }
            umma_commit(&bar[kBarFinalO]);
            mbar_wait(&bar[kBarFinalO], 0);
        }
        __syncwarp();
    } else if (warp < kAttnSoftmaxWarps) {
        // ================================== softmax (token / thread, half the rows / warp)
        // The two row halves share no running max, sum or O^T column, so each
        // half (one warp per TMEM lane quadrant) votes and syncs on its own.
        constexpr int kH = NR / 2;                            // rows per thread
        constexpr int kSm = 32 * kAttnSoftmaxWarps / 2;       // softmax threads of a row half
        const int q = warp & 3;                               // TMEM lane quadrant
        const int r0 = (warp >> 2) * kH;                      // first row of this warp
        const uint32_t nb_sync = r0 == 0 ? kNbSoftmax : kNbSoftmaxHi;
        const uint32_t nb_vote = r0 == 0 ? kNbSoftmaxVote : kNbSoftmaxVoteHi;
        const int tok = 32 * q + lane;                        // token of the tile this thread owns
        const int myslot = tok >> 4, mytok = tok & 15;
        const float inv_scale = 1.f / scale_log2;             // thresholds in raw-score units
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        int pos = 0;
        for (int p = 0;; ++p) {
            const int pb = p & 1;
            cta_wait(&bar[kBarLFull + pb], (p >> 1) & 1, s_abort);
            const int* info = s_info + pb * kAttnInfoInts;
            const int n = info[0];
            if (named_bar_or(nb_vote, kSm, n < 0 || *s_abort)) break;
            // the epilogue of chunk p-2 has read this buffer's running max and sums
            if (p >= 2) cta_wait(&bar[kBarOFree + pb], ((p >> 1) - 1) & 1, s_abort);
            // running max m (log2 units) and the raw-score threshold (m + 32) / scale of
            // every row, set from the chunk's first valid token at its first tile; rows
            // past the real ones have both at +inf, so their scores never vote and their
            // probabilities are 0 (the padded columns are never read)
            float* mr = s_m + pb * 64;
            float* thr = s_thr + pb * 64;
            if (q == 0 && lane < kH && r0 + lane >= rows) {
                const float kPosInf = __int_as_float(0x7f800000);
                mr[r0 + lane] = thr[r0 + lane] = kPosInf;
            }
            float l[kH];                                      // this token's share of its rows' sums
#pragma unroll
            for (int r = 0; r < kH; ++r) l[r] = 0.f;
            for (int i = 0; i < n; ++i, ++pos) {
                const int st = pos & 1;
                const int* e = info + 8 + 4 * i;
                const int nvj = (static_cast<uint32_t>(myslot < 4 ? e[1] : e[2]) >> (8 * (myslot & 3))) & 0xFF;
                const bool valid = mytok < nvj;
                cta_wait(&bar[kBarSFull + st], (pos >> 1) & 1, s_abort);
                __syncwarp();                                 // tcgen05.ld is warp-wide: lanes together
                tc_fence_after_sync();
                float x[kH];                                  // raw scores q.k of this token, rows r0..
                if constexpr (kH == 16) {
                    uint32_t v[16];
                    tmem_ld_x16(tmem + lane_base + st * 64 + r0, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int r = 0; r < 16; ++r) x[r] = __uint_as_float(v[r]);
                } else {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + st * 64 + r0, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int r = 0; r < 32; ++r) x[r] = __uint_as_float(v[r]);
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar[kBarSFree + st]);
                if (i == 0) {
                    // seed the running max: the first token of the tile's first occupied slot
                    const uint64_t nvs = static_cast<uint32_t>(e[1]) | (static_cast<uint64_t>(static_cast<uint32_t>(e[2])) << 32);
                    const int j0 = (__ffsll(static_cast<long long>(nvs)) - 1) >> 3;
                    if (tok == kBlockTokens * j0) {
#pragma unroll
                        for (int r = 0; r < kH; ++r)
                            if (r0 + r < rows) {
                                const float m0 = x[r] * scale_log2;
                                mr[r0 + r] = m0;
                                thr[r0 + r] = (m0 + kAttnLazy) * inv_scale;
                            }
                    }
                    named_bar_sync(nb_sync, kSm);
                }
                // does any row's running max move (by more than 2^32)?
                bool up = false;
                if (valid) {
#pragma unroll
                    for (int r = 0; r < kH; r += 4) {
                        const float4 t4 = *reinterpret_cast<const float4*>(thr + r0 + r);
                        up |= (x[r] > t4.x) | (x[r + 1] > t4.y) | (x[r + 2] > t4.z) | (x[r + 3] > t4.w);
                    }
                }
                if (named_bar_or(nb_vote, kSm, up)) {
                    // tile maxima (log2 units): lane r of each warp keeps row r0 + r of its tokens
                    float mine = kNegInf;
#pragma unroll
                    for (int r = 0; r < kH; ++r) {
                        const float wm = warp_max_f32((valid && r0 + r < rows) ? x[r] * scale_log2 : kNegInf);
                        if (lane == r) mine = wm;
                    }
                    if (lane < kH) s_wmax[q * 64 + r0 + lane] = mine;
                    named_bar_sync(nb_sync, kSm);
                    if (q == 0 && lane < kH) {                // warps 0 and 4: their rows
                        const int r = r0 + lane;
                        const float tmx = fmaxf(fmaxf(s_wmax[r], s_wmax[64 + r]), fmaxf(s_wmax[128 + r], s_wmax[192 + r]));
                        const float mo = mr[r];
                        float a = 1.f;
                        if (r < rows && tmx > mo + kAttnLazy) {
                            a = attn_exp2(mo - tmx);
                            mr[r] = tmx;
                            thr[r] = (tmx + kAttnLazy) * inv_scale;
                        }
                        s_alpha[r] = a;
                    }
                    named_bar_sync(nb_sync, kSm);
#pragma unroll
                    for (int r = 0; r < kH; ++r) l[r] *= s_alpha[r0 + r];
                    if (i > 0) {
                        // the previous tile's product must have landed in O^T before it is rescaled
                        cta_wait(&bar[kBarPFree + (pos - 1) % kPBufs], ((pos - 1) / kPBufs) & 1, s_abort);
                        __syncwarp();
                        tc_fence_after_sync();
#pragma unroll
                        for (int part = 0; part < 2 * kH / 16; ++part) {   // head and remainder columns
                            const int c0 = (part & (kH / 16 - 1)) * 16;           // column within the half
                            const uint32_t oaddr = tmem + lane_base + kOCol + pb * kOStride +
                                                   (part >= kH / 16 ? NR : 0) + r0 + c0;
                            uint32_t o[16];
                            tmem_ld_x16(oaddr, o);
                            tmem_ld_wait();
#pragma unroll
                            for (int r = 0; r < 16; ++r)
                                o[r] = __float_as_uint(__uint_as_float(o[r]) * s_alpha[r0 + c0 + r]);
                            tmem_st_x16(oaddr, o);
                        }
                        tmem_st_wait();
                    }
                }
                // this token's probabilities for this warp's rows as bf16 head and
                // remainder words, computed before the wait for the product that last
                // read this P^T buffer (with one buffer, the previous tile's), so the
                // exponentials overlap that product; the words of rows r..r+7 replace
                // their scores in x (head words first, then remainder words)
                if (valid) {
#pragma unroll
                    for (int c8 = 0; c8 < kH / 8; ++c8) {
                        const int r = 8 * c8;
                        const float4 ma = *reinterpret_cast<const float4*>(mr + r0 + r);
                        const float4 mb = *reinterpret_cast<const float4*>(mr + r0 + r + 4);
                        const float p0 = attn_exp2(fmaf(x[r + 0], scale_log2, -ma.x));
                        const float p1 = attn_exp2(fmaf(x[r + 1], scale_log2, -ma.y));
                        const float p2 = attn_exp2(fmaf(x[r + 2], scale_log2, -ma.z));
                        const float p3 = attn_exp2(fmaf(x[r + 3], scale_log2, -ma.w));
                        const float p4 = attn_exp2(fmaf(x[r + 4], scale_log2, -mb.x));
                        const float p5 = attn_exp2(fmaf(x[r + 5], scale_log2, -mb.y));
                        const float p6 = attn_exp2(fmaf(x[r + 6], scale_log2, -mb.z));
                        const float p7 = attn_exp2(fmaf(x[r + 7], scale_log2, -mb.w));
                        l[r + 0] += p0;
                        l[r + 1] += p1;
                        l[r + 2] += p2;
                        l[r + 3] += p3;
                        l[r + 4] += p4;
                        l[r + 5] += p5;
                        l[r + 6] += p6;
                        l[r + 7] += p7;
                        const uint32_t h01 = pack_bf16x2(p0, p1), h23 = pack_bf16x2(p2, p3);
                        const uint32_t h45 = pack_bf16x2(p4, p5), h67 = pack_bf16x2(p6, p7);
                        x[r + 0] = __uint_as_float(h01);
                        x[r + 1] = __uint_as_float(h23);
                        x[r + 2] = __uint_as_float(h45);
                        x[r + 3] = __uint_as_float(h67);
                        x[r + 4] = __uint_as_float(pack_bf16x2(p0 - bf16_lo(h01), p1 - bf16_hi(h01)));
                        x[r + 5] = __uint_as_float(pack_bf16x2(p2 - bf16_lo(h23), p3 - bf16_hi(h23)));
                        x[r + 6] = __uint_as_float(pack_bf16x2(p4 - bf16_lo(h45), p5 - bf16_hi(h45)));
                        x[r + 7] = __uint_as_float(pack_bf16x2(p6 - bf16_lo(h67), p7 - bf16_hi(h67)));
                    }
                }
                const int pbuf = pos % kPBufs;
                if (pos >= kPBufs) cta_wait(&bar[kBarPFree + pbuf], ((pos / kPBufs) - 1) & 1, s_abort);
                uint8_t* prow = sP + pbuf * kPBufBytes + tok * 128;
                if (valid) {
#pragma unroll
                    for (int c8 = 0; c8 < kH / 8; ++c8) {
                        const int cg = r0 / 8 + c8;                           // 16-B chunk of the row
                        const int off = (cg ^ (tok & 7)) << 4;
                        const int roff = NR == 32 ? (((cg + 4) ^ (tok & 7)) << 4) : kAttnHalf + off;
                        const int r = 8 * c8;
                        *reinterpret_cast<uint4*>(prow + off) =
                            make_uint4(__float_as_uint(x[r]), __float_as_uint(x[r + 1]),
                                       __float_as_uint(x[r + 2]), __float_as_uint(x[r + 3]));
                        *reinterpret_cast<uint4*>(prow + roff) =
                            make_uint4(__float_as_uint(x[r + 4]), __float_as_uint(x[r + 5]),
                                       __float_as_uint(x[r + 6]), __float_as_uint(x[r + 7]));
                    }
                } else {
                    // a token past the context or in a free slot: zero weights; in an occupied
                    // slot its value row reads as zero too (zero times a stale non-finite
                    // value is not zero)
#pragma unroll
                    for (int c8 = 0; c8 < kH / 8; ++c8) {
                        const int cg = r0 / 8 + c8;
                        const int off = (cg ^ (tok & 7)) << 4;
                        const int roff = NR == 32 ? (((cg + 4) ^ (tok & 7)) << 4) : kAttnHalf + off;
                        *reinterpret_cast<uint4*>(prow + off) = make_uint4(0u, 0u, 0u, 0u);
                        *reinterpret_cast<uint4*>(prow + roff) = make_uint4(0u, 0u, 0u, 0u);
                    }
                    if (nvj > 0 && r0 == 0) {
                        cta_wait(&bar[kBarVFull + st], (pos >> 1) & 1, s_abort);   // orders the copy first
                        uint8_t* vrow = sV + st * kAttnStageBytes + tok * 128;
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            *reinterpret_cast<uint4*>(vrow + 16 * k) = make_uint4(0u, 0u, 0u, 0u);
                            *reinterpret_cast<uint4*>(vrow + kAttnHalf + 16 * k) = make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar[kBarPFull + pbuf]);
            }
            // the chunk's row sums over this warp's tokens: lane r gets row r0 + r
            float* lw = s_lw + (pb * 4 + q) * 64 + r0;
            float sum;
            if constexpr (kH == 16)
                sum = warp_reduce_scatter16<false>(l, lane);
            else
                sum = warp_reduce_scatter32<false>(l, lane);
            if (lane < kH) lw[lane] = sum;
            if (NR == 32 && r0 == 0) lw[32 + lane] = 0.f;                  // unused rows
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bar[kBarSMDone + pb]);
                mbar_arrive(&bar[kBarLFree + pb]);
            }
        }
    } else {
        // ============================================ epilogue (channel / thread)
        const int q = warp & 3;                               // TMEM lane quadrant
        const int chn = 32 * q + lane;                        // head-dimension channel
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        const bool leader = warp == kAttnEpiWarp && lane == 0;
        for (int p = 0;; ++p) {
            const int pb = p & 1;
            cta_wait(&bar[kBarLFull + pb], (p >> 1) & 1, s_abort);
            const int* info = s_info + pb * kAttnInfoInts;
            const int n = info[0], c = info[1], u = info[2], ncu = info[3];
            const bool stop = named_bar_or(kNbEpiVote, 128, n < 0 || *s_abort);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[kBarLFree + pb]);
            if (stop) break;
            cta_wait(&bar[kBarSMDone + pb], (p >> 1) & 1, s_abort);
            cta_wait(&bar[kBarODone + pb], (p >> 1) & 1, s_abort);
            tc_fence_after_sync();
            float* f_inv = s_fin + pb * 64;
            float* f_lse = s_fin + 128 + pb * 64;
            if (q < 2) {
                const int r = 32 * q + lane;
                const float* lw = s_lw + pb * 4 * 64;
                const float L = (lw[r] + lw[64 + r]) + (lw[128 + r] + lw[192 + r]);
                f_inv[r] = L > 0.f ? 1.f / L : 0.f;
                f_lse[r] = L > 0.f ? s_m[pb * 64 + r] + log2f(L) : kNegInf;
            }
            named_bar_sync(kNbEpi, 128);                      // 1/sum and lse ready; m and sums read
            const int b = u / d.Hkv, h = u - b * d.Hkv;
            const bool direct = ncu == 1;
            float* dst = ws_o + static_cast<long long>(c) * rows * kHeadDim;
            // O^T, 32 rows at a time: head + remainder products of this thread's channel
#pragma unroll
            for (int hh = 0; hh < NR / 32; ++hh) {
                uint32_t v[32];
                float o[32];
                if (n > 0) {
                    tmem_ld_32x32b_x32(tmem + lane_base + kOCol + pb * kOStride + 32 * hh, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int r = 0; r < 32; ++r) o[r] = __uint_as_float(v[r]);
                    tmem_ld_32x32b_x32(tmem + lane_base + kOCol + pb * kOStride + NR + 32 * hh, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int r = 0; r < 32; ++r) o[r] += __uint_as_float(v[r]);
                } else {
#pragma unroll
                    for (int r = 0; r < 32; ++r) o[r] = 0.f;
                }
#pragma unroll
                for (int rr = 0; rr < 32; ++rr) {
                    const int r = 32 * hh + rr;
                    if (r >= rows) break;
                    if (direct) {
                        const long long orow = (static_cast<long long>(b) * d.Qn + r / G) * d.Hq + h * G + r % G;
                        out[orow * kHeadDim + chn] = o[rr] * f_inv[r];
                    } else {
                        dst[r * kHeadDim + chn] = o[rr] * f_inv[r];
                    }
                }
            }
            tc_fence_before_sync();
            named_bar_sync(kNbEpi, 128);                      // every thread has read its O^T
            if (leader) mbar_arrive(&bar[kBarOFree + pb]);
            if (direct) {
                if (q < 2 && 32 * q + lane < rows) {
                    const int r = 32 * q + lane;
                    const long long orow = (static_cast<long long>(b) * d.Qn + r / G) * d.Hq + h * G + r % G;
                    lse_out[orow] = f_lse[r] * kLn2;
                }
            } else {
                if (q < 2 && 32 * q + lane < rows) ws_lse[static_cast<long long>(c) * rows + 32 * q + lane] = f_lse[32 * q + lane];
                __threadfence();
                named_bar_sync(kNbEpi, 128);
                if (leader) *s_last = atomicAdd(ws_ticket + u, 1) == ncu - 1 ? 1 : 0;
                named_bar_sync(kNbEpi, 128);
                if (*s_last) {
                    // merge the unit's partials: out = sum_j 2^(lse_j - M) o_j / sum_j 2^(lse_j - M).
                    // Thread r < rows turns row r's log2-sum-exps into weights, then every
                    // thread (one channel) sums the weighted partials, loads in flight together.
                    __threadfence();
                    const long long c0 = static_cast<long long>(u) * ncu;
                    const int t = 32 * q + lane;
                    if (t < rows) {
                        float lj[kAttnMaxChunks];
                        float M = kNegInf;
#pragma unroll
                        for (int jj = 0; jj < kAttnMaxChunks; ++jj) {
                            lj[jj] = jj < ncu ? __ldcg(ws_lse + (c0 + jj) * rows + t) : kNegInf;
                            M = fmaxf(M, lj[jj]);
                        }
                        float L = 0.f;
#pragma unroll
                        for (int jj = 0; jj < kAttnMaxChunks; ++jj) {
                            lj[jj] = (M != kNegInf && lj[jj] != kNegInf) ? exp2f(lj[jj] - M) : 0.f;   // empty partial: 0
                            L += lj[jj];
                        }
                        const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
                        for (int jj = 0; jj < kAttnMaxChunks; ++jj) s_mw[t * kAttnMaxChunks + jj] = lj[jj] * inv;
                        const long long orow = (static_cast<long long>(b) * d.Qn + t / G) * d.Hq + h * G + t % G;
                        lse_out[orow] = L > 0.f ? (M + log2f(L)) * kLn2 : kNegInf;
                    }
                    named_bar_sync(kNbEpi, 128);
                    // 32 threads per row (4 channels each), 4 rows per pass: up to 8 float4
                    // loads in flight per thread
                    const int et = 32 * q + lane;
                    const int rsub = et >> 5, c4 = (et & 31) * 4;
                    for (int r0 = 0; r0 < rows; r0 += 4) {
                        float4 xv[1][kAttnMaxChunks];
#pragma unroll
                        for (int s2 = 0; s2 < 1; ++s2) {
                            const int r = r0 + 4 * s2 + rsub;
#pragma unroll
                            for (int jj = 0; jj < kAttnMaxChunks; ++jj)
                                xv[s2][jj] = (r < rows && jj < ncu)
                                                 ? __ldcg(reinterpret_cast<const float4*>(
                                                       ws_o + ((c0 + jj) * rows + r) * kHeadDim + c4))
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
                        }
#pragma unroll
                        for (int s2 = 0; s2 < 1; ++s2) {
                            const int r = r0 + 4 * s2 + rsub;
                            if (r >= rows) continue;
                            const float* w = s_mw + r * kAttnMaxChunks;
                            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                            for (int jj = 0; jj < kAttnMaxChunks; ++jj) {
                                acc.x += w[jj] * xv[s2][jj].x;
                                acc.y += w[jj] * xv[s2][jj].y;
                                acc.z += w[jj] * xv[s2][jj].z;
                                acc.w += w[jj] * xv[s2][jj].w;
                            }
                            const long long orow = (static_cast<long long>(b) * d.Qn + r / G) * d.Hq + h * G + r % G;
                            *reinterpret_cast<float4*>(out + orow * kHeadDim + c4) = acc;
                        }
                    }
                    if (leader) ws_ticket[u] = 0;             // ready for the next call
                }
            }
        }
    }

    // ---------------------------------------------------------- teardown
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == kAttnSWarp) tmem_dealloc(tmem, kAttnTmemCols);
    if (tid == 0) {
        // the last CTA out resets the chunk counter for the next call
        __threadfence();
        if (atomicAdd(ws_sched + 1, 1) == static_cast<int>(gridDim.x) - 1) {
            atomicExch(ws_sched, 0);
            atomicExch(ws_sched + 1, 0);
        }
    }
}

}  // namespace oasis
