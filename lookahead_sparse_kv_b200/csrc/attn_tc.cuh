// attn_tc.cuh - sparse GQA decode attention on the 5th-generation tensor
// cores (tcgen05, TMEM accumulators).
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching, Figure 7 (right): one attention kernel runs the normal and
// the draft queries together over the sparse KV working set; Figure 9: the
// per-head slot table names the block each pool slot holds.
//
// Work split (stream-K): the B*Hkv*K pool slots are cut into one contiguous
// range per CTA (one CTA per SM).  A CTA walks the occupied slots of its
// range in tiles of up to 8 slots (128 tokens) of one (sequence, KV head)
// unit.  Every softmax group writes one normalised partial (output +
// log-sum-exp) per unit of the range; attn_merge_kernel combines them.
//
// Per tile, with NQ >= Qn*G query columns (32 or 64):
//   S^T[128 tok x NQ]   = K . Q^T                    (8 x tcgen05.mma, K = 16)
//   P^T                 = exp2(S^T * scale*log2e - m_ref), as a bf16 head and
//                         a bf16 remainder (the weights keep ~16 bits)
//   O^T[128 d x 2NQ]   += V^T . [P_head | P_rest]^T  (V and P^T read MN-major;
//                         output = head columns + rest columns)
// The per-column reference max m_ref only moves when a tile exceeds it by
// 2^8; then O^T in TMEM and the column sums are rescaled.
//
// Roles (12 warps):
//   warp 0   TMA producer: the K half [128 tok x 128 d] of each tile into a
//            2-deep ring, the V half into a 3-deep ring (2 for NQ = 64):
//            K is free again once S^T is computed, V only after the PV
//            product, so K runs further ahead.  A run of 8 consecutive slots
//            is one 3-D box per 64-column half; otherwise one 2-D box per
//            slot and half (128-byte swizzle, L2 evict-first).
//   warp 1   S^T issuer (one thread).
//   warp 2   PV issuer (one thread).
//   warp 3   Q loader: the unit's Qn*G query rows, swizzled K-major, into a
//            double buffer, one unit ahead.
//   warps 4-11  softmax.  NQ = 32: two groups of 4 warps (one per TMEM lane
//            quadrant = 32 token rows), even tiles to group 0 and odd tiles to
//            group 1, each with its own P^T buffer and O^T accumulator, so the
//            two tiles' softmax and PV products overlap.  NQ = 64: one group
//            of 8 warps (two column halves).  A thread owns one token row and
//            32 query columns; at a unit end it owns one channel row of O^T.
#pragma once

#include "attn.cuh"
#include "common.cuh"

namespace oasis {

constexpr int kTcTileSlots = 8;
constexpr int kTcRegion = 128 * 128;                 // 128 rows x 128 B (64 bf16 columns)
constexpr int kTcHalfBytes = 2 * kTcRegion;          // one K or V tile: [lo 64 | hi 64] columns
constexpr int kTcList = 512;                         // occupied slots listed per CTA
constexpr int kTcFirstSoftWarp = 4;
constexpr int kTcSoftWarps = 8;
constexpr int kTcThreads = 32 * (kTcFirstSoftWarp + kTcSoftWarps);
constexpr int kTcTmemCols = 256;                     // S^T x2 at 0/64, O^T per group from 128
constexpr int kTcKBufs = 2;

// Shared-memory layout for NQ query columns.
template <int NQ>
struct TcSmem {
    static constexpr int kGroups = NQ <= 32 ? 2 : 1;
    static constexpr int kHalves = NQ / 32;                          // column halves per group
    static constexpr int kGroupThreads = 128 * kHalves;
    static constexpr int kVBufs = NQ <= 32 ? 3 : 2;
    static constexpr int kK = 0;
    static constexpr int kV = kK + kTcKBufs * kTcHalfBytes;
    static constexpr int kQ = kV + kVBufs * kTcHalfBytes;
    static constexpr int kQRegion = NQ * 128;                        // NQ rows x 128 B
    static constexpr int kQBuf = 2 * kQRegion;
    static constexpr int kPAtoms = (2 * NQ + 63) / 64;               // P^T: 2NQ columns, 64 per atom
    static constexpr int kP = kQ + 2 * kQBuf;
    static constexpr int kPBuf = kPAtoms * kTcRegion;
    static constexpr int kListSlot = kP + kGroups * kPBuf;
    static constexpr int kListNv = kListSlot + kTcList * 4;
    static constexpr int kListUnit = kListNv + kTcList * 4;
    static constexpr int kRed = kListUnit + kTcList * 4;             // [groups][4][64] floats
    static constexpr int kMref = kRed + kGroups * 256 * 4;           // [groups][64]
    static constexpr int kAlpha = kMref + kGroups * 64 * 4;
    static constexpr int kLtot = kAlpha + kGroups * 64 * 4;
    static constexpr int kMisc = kLtot + kGroups * 64 * 4;           // 32 ints
    static constexpr int kBars = kMisc + 32 * 4;
    static constexpr int kBytes = kBars + 24 * 8 + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
    static_assert(128 + kGroups * 2 * NQ <= kTcTmemCols, "TMEM budget");
};

// mbarrier indices
enum {
    kBarKFull = 0,    // [2]
    kBarKEmpty = 2,   // [2]
    kBarVFull = 4,    // [3]
    kBarVEmpty = 7,   // [3]
    kBarSFull = 10,   // [2]
    kBarSEmpty = 12,  // [2]
    kBarPFull = 14,   // [2] per group
    kBarPEmpty = 16,  // [2] per group
    kBarQFull = 18,   // [2]
    kBarQEmpty = 20,  // [2]
    kBarCount = 22
};

__device__ __forceinline__ uint64_t umma_desc_sw128_mn(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(lbo >> 4) << 16;      // stride between 64-element atoms along M/N
    d |= static_cast<uint64_t>(sbo >> 4) << 32;      // stride between 8-row groups along K
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

__device__ __forceinline__ void tmem_ld_x32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Named barrier of one softmax group (ids 1 and 2; 0 is __syncthreads).
__device__ __forceinline__ void group_bar(int g, int n_threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "r"(n_threads) : "memory");
}

// End of the tile that starts at list entry i: up to 8 entries of one unit
// (l_unit holds each listed slot's unit, so no role divides in its loop).
__device__ __forceinline__ int tc_tile_end(const int* l_unit, int i, int n) {
    const int u = l_unit[i];
    int j = i + 1;
    while (j < n && j - i < kTcTileSlots && l_unit[j] == u) ++j;
    return j;
}

// NQ: query columns of the S^T product (Qn*G rows padded to 32 or 64).
// Partial p = groups * (cta + unit) + group of ws_o / ws_lse.
template <int NQ>
__global__ void __launch_bounds__(kTcThreads, 1)
    sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_pool16, const __grid_constant__ CUtensorMap tm_pool3d,
                          Dims d, const uint16_t* __restrict__ q,
                          const int32_t* __restrict__ slot_table, const int32_t* __restrict__ ctx_len,
                          float scale_log2, float* __restrict__ ws_o, float* __restrict__ ws_lse) {
    using TS = TcSmem<NQ>;
    constexpr int NG = TS::kGroups;
    constexpr int kVBufs = TS::kVBufs;
    constexpr int NH = 32;                               // query columns per softmax thread
    const float kNegInf = -__int_as_float(0x7f800000);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int* l_slot = reinterpret_cast<int*>(sm + TS::kListSlot);
    int* l_nv = reinterpret_cast<int*>(sm + TS::kListNv);
    int* l_unit = reinterpret_cast<int*>(sm + TS::kListUnit);
    // s_misc: [0] list count, [1] abort flag, [2..5] per-tile abort snapshots
    // [parity][group], [6..7] final snapshots [group], [8..23] rescale votes
    // [parity][softmax warp].  Per-tile slots alternate with the group's tile
    // parity: a warp can only rewrite a slot after the next group barrier,
    // which every warp reaches after reading the slot.
    int* s_misc = reinterpret_cast<int*>(sm + TS::kMisc);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + TS::kBars);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);
    volatile int* abort_flag = s_misc + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = d.G();
    const int rows = d.Qn * G;
    const long long K = d.K;
    const long long T = static_cast<long long>(d.B) * d.Hkv * K;
    const long long NS = gridDim.x;
    const long long cs = static_cast<long long>(blockIdx.x);
    const long long c_begin = (cs * T + NS - 1) / NS;
    const long long c_end = ((cs + 1) * T + NS - 1) / NS;

    // ---- occupied slots of the range, in slot order (warp 0), barriers, TMEM
    if (warp == 0) {
        int n = 0;
        for (long long base = c_begin; base < c_end; base += 32) {
            const long long s = base + lane;
            int nv = 0, unit = 0;
            if (s < c_end) {
                // slot indices stay below 2^26 (host check), so 32-bit division
                unit = static_cast<int>(static_cast<unsigned>(s) / static_cast<unsigned>(K));
                int blk = slot_table[s];
                if (blk < -1 || blk >= d.N) {
                    raise_dev_error(OASIS_DEVERR_ID_RANGE);
                    blk = -1;
                }
                if (blk >= 0) nv = min(kBlockTokens, ctx_len[unit / d.Hkv] - blk * kBlockTokens);
            }
            const unsigned m = __ballot_sync(0xFFFFFFFFu, nv > 0);
            if (nv > 0) {
                const int pos = n + __popc(m & ((1u << lane) - 1u));
                l_slot[pos] = static_cast<int>(s);
                l_nv[pos] = nv;
                l_unit[pos] = unit;
            }
            n += __popc(m);
        }
        if (lane == 0) {
            s_misc[0] = n;
            s_misc[1] = 0;
            for (int b = 0; b < kBarCount; ++b) {
                const bool by_softmax = (b >= kBarSEmpty && b < kBarSEmpty + 2) || (b >= kBarPFull && b < kBarPFull + 2);
                mbar_init(&bars[b], by_softmax ? static_cast<uint32_t>(4 * TS::kHalves) : 1u);
            }
        }
        fence_mbar_init();
    } else if (warp == 1) {
        tmem_alloc(tmem_slot, kTcTmemCols);
        tmem_relinquish();
    } else if (warp >= kTcFirstSoftWarp) {
        // zero the V ring and the P^T buffers: rows of tile positions that no
        // slot fills must hold finite values (they meet P = 0)
        const int st = tid - 32 * kTcFirstSoftWarp;
        for (int i = st; i < kVBufs * kTcHalfBytes / 16; i += 32 * kTcSoftWarps)
            reinterpret_cast<uint4*>(sm + TS::kV)[i] = make_uint4(0, 0, 0, 0);
        for (int i = st; i < NG * TS::kPBuf / 16; i += 32 * kTcSoftWarps)
            reinterpret_cast<uint4*>(sm + TS::kP)[i] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const int n_list = s_misc[0];
    const uint32_t tmem = *tmem_slot;
    const uint32_t sm_base = smem_addr(sm);
    const long long u_first = c_begin < c_end ? c_begin / K : 0;
    const long long u_last = c_begin < c_end ? (c_end - 1) / K : -1;

    if (warp == 0) {
        // ===================== TMA producer =====================
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            prefetch_tensormap(&tm_pool16);
            prefetch_tensormap(&tm_pool3d);
            for (int i = 0, t = 0; i < n_list; ++t) {
                const int e = tc_tile_end(l_unit, i, n_list);
                const int kb = t & 1, vb = t % kVBufs;
                // a full run of 8 consecutive slots: one box per half
                const bool run = e - i == kTcTileSlots && l_slot[e - 1] - l_slot[i] == kTcTileSlots - 1;
                bool ok = t < kTcKBufs || mbar_wait(&bars[kBarKEmpty + kb], ((t >> 1) - 1) & 1);
                if (ok && !*abort_flag) {
                    uint64_t* full = &bars[kBarKFull + kb];
                    uint8_t* dst = sm + TS::kK + kb * kTcHalfBytes;
                    if (run) {
                        mbar_arrive_expect_tx(full, kTcHalfBytes);
                        tma_load_3d(dst, &tm_pool3d, full, 0, 0, l_slot[i], pol);
                        tma_load_3d(dst + kTcRegion, &tm_pool3d, full, 64, 0, l_slot[i], pol);
                    } else {
                        mbar_arrive_expect_tx(full, (e - i) * (kBlockBytes / 2));
                        for (int j = 0; j < e - i; ++j) {
                            const int y = l_slot[i + j] * (2 * kBlockTokens);
                            tma_load_2d(dst + j * 2048, &tm_pool16, full, 0, y, pol);
                            tma_load_2d(dst + kTcRegion + j * 2048, &tm_pool16, full, 64, y, pol);
                        }
                    }
                }
                ok = ok && (t < kVBufs || mbar_wait(&bars[kBarVEmpty + vb], ((t / kVBufs) - 1) & 1));
                if (!ok) {
                    raise_dev_error(OASIS_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                }
                if (*abort_flag) break;
                uint64_t* full = &bars[kBarVFull + vb];
                uint8_t* dst = sm + TS::kV + vb * kTcHalfBytes;
                if (run) {
                    mbar_arrive_expect_tx(full, kTcHalfBytes);
                    tma_load_3d(dst, &tm_pool3d, full, 0, kBlockTokens, l_slot[i], pol);
                    tma_load_3d(dst + kTcRegion, &tm_pool3d, full, 64, kBlockTokens, l_slot[i], pol);
                } else {
                    mbar_arrive_expect_tx(full, (e - i) * (kBlockBytes / 2));
                    for (int j = 0; j < e - i; ++j) {
                        const int y = l_slot[i + j] * (2 * kBlockTokens) + kBlockTokens;
                        tma_load_2d(dst + j * 2048, &tm_pool16, full, 0, y, pol);
                        tma_load_2d(dst + kTcRegion + j * 2048, &tm_pool16, full, 64, y, pol);
                    }
                }
                i = e;
            }
        }
    } else if (warp == 1) {
        // ===================== S^T issuer =====================
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16_f32(128, NQ);
            int ui = -1, last_t = -1;
            bool ok = true;
            for (int i = 0, t = 0; i < n_list; ++t) {
                const int e = tc_tile_end(l_unit, i, n_list);
                const int b = t & 1;
                if (i == 0 || l_unit[i] != l_unit[i - 1]) {
                    ++ui;
                    ok = mbar_wait(&bars[kBarQFull + (ui & 1)], (ui >> 1) & 1);
                }
                ok = ok && mbar_wait(&bars[kBarKFull + b], (t >> 1) & 1);
                ok = ok && (t < 2 || mbar_wait(&bars[kBarSEmpty + b], ((t >> 1) - 1) & 1));
                if (!ok || *abort_flag) break;
                tc_fence_after_sync();
                const uint32_t kbase = sm_base + TS::kK + b * kTcHalfBytes;
                const uint32_t qbase = sm_base + TS::kQ + (ui & 1) * TS::kQBuf;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t ad = umma_desc_sw128(kbase + (ks >> 2) * kTcRegion + (ks & 3) * 32);
                    const uint64_t bd = umma_desc_sw128(qbase + (ks >> 2) * TS::kQRegion + (ks & 3) * 32);
                    umma_bf16(tmem + b * 64, ad, bd, idesc, ks > 0);
                }
                umma_commit(&bars[kBarSFull + b]);
                umma_commit(&bars[kBarKEmpty + b]);
                if (e == n_list || l_unit[e] != l_unit[i]) umma_commit(&bars[kBarQEmpty + (ui & 1)]);
                last_t = t;
                i = e;
            }
            if (!ok) {
                raise_dev_error(OASIS_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            // products in flight must finish before TMEM is released
            if (last_t >= 0) mbar_wait(&bars[kBarSFull + (last_t & 1)], (last_t >> 1) & 1);
        }
    } else if (warp == 2) {
        // ===================== PV issuer =====================
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16_f32(128, 2 * NQ) | (1u << 15) | (1u << 16);
            int last_unit[2] = {-1, -1};
            int last_t = -1;
            bool ok = true;
            for (int i = 0, t = 0; i < n_list; ++t) {
                const int e = tc_tile_end(l_unit, i, n_list);
                const int g = NG == 2 ? (t & 1) : 0;
                const int n_g = NG == 2 ? (t >> 1) : t;
                const int vb = t % kVBufs;
                ok = mbar_wait(&bars[kBarPFull + g], n_g & 1) && mbar_wait(&bars[kBarVFull + vb], (t / kVBufs) & 1);
                if (!ok || *abort_flag) break;
                tc_fence_after_sync();
                const bool first = last_unit[g] != l_unit[i];
                last_unit[g] = l_unit[i];
                const uint32_t vbase = sm_base + TS::kV + vb * kTcHalfBytes;
                const uint32_t pbase = sm_base + TS::kP + g * TS::kPBuf;
                const uint32_t o_col = 128 + g * 2 * NQ;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint64_t ad = umma_desc_sw128_mn(vbase + k * 2048, kTcRegion, 1024);
                    const uint64_t bd = umma_desc_sw128_mn(pbase + k * 2048, kTcRegion, 1024);
                    umma_bf16(tmem + o_col, ad, bd, idesc, (first && k == 0) ? 0u : 1u);
                }
                umma_commit(&bars[kBarVEmpty + vb]);
                umma_commit(&bars[kBarPEmpty + g]);
                last_t = t;
                i = e;
            }
            if (!ok) {
                raise_dev_error(OASIS_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            if (last_t >= 0) {
                const int g = NG == 2 ? (last_t & 1) : 0;
                const int n_g = NG == 2 ? (last_t >> 1) : last_t;
                mbar_wait(&bars[kBarPEmpty + g], n_g & 1);
            }
        }
    } else if (warp == 3) {
        // ===================== Q loader =====================
        // rows r = j*G + g of the unit's query block, K-major, 128-byte
        // swizzle: two regions (channels 0-63, 64-127) of NQ rows x 128 B
        int ui = 0;
        for (int i = 0; i < n_list; ++i) {
            if (i > 0 && l_unit[i] == l_unit[i - 1]) continue;
            const int qb = ui & 1;
            const bool ok = __all_sync(0xFFFFFFFFu, ui < 2 || mbar_wait(&bars[kBarQEmpty + qb], ((ui >> 1) - 1) & 1));
            if (!ok) {
                if (lane == 0) {
                    raise_dev_error(OASIS_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                }
                break;
            }
            if (__any_sync(0xFFFFFFFFu, *abort_flag != 0)) break;
            const int u = l_unit[i];
            const int b = u / d.Hkv, h = u % d.Hkv;
            uint8_t* qdst = sm + TS::kQ + qb * TS::kQBuf;
            for (int it = lane; it < NQ * 16; it += 32) {
                const int qr = it >> 4, c = it & 15;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (qr < rows)
                    v = *reinterpret_cast<const uint4*>(
                        q + ((static_cast<long long>(b) * d.Qn + qr / G) * d.Hq + h * G + qr % G) * kHeadDim + c * 8);
                const int region = c >> 3, cc = c & 7;
                const int off = (qr >> 3) * 1024 + (qr & 7) * 128 + ((cc ^ (qr & 7)) << 4);
                *reinterpret_cast<uint4*>(qdst + region * TS::kQRegion + off) = v;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kBarQFull + qb]);
            ++ui;
        }
    } else {
        // ===================== softmax groups =====================
        const int sw = warp - kTcFirstSoftWarp;                 // 0..7
        const int quad = warp & 3;                              // TMEM lane quadrant this warp may access
        const int g = NG == 2 ? (sw >> 2) : 0;
        const int half = NG == 2 ? 0 : (sw >> 2);
        const int cb = half * NH;                               // first query column of this thread
        const int gt = (NG == 2 ? (sw & 3) : sw) * 32 + lane;   // thread index in the group
        const int gw0 = NG == 2 ? 4 * g : 0;                    // first softmax warp of the group
        constexpr int kGW = 4 * TS::kHalves;                    // warps per group
        const int r = quad * 32 + lane;                         // token row of a tile; channel row of O^T
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t o_col = 128 + g * 2 * NQ;
        float* s_red = reinterpret_cast<float*>(sm + TS::kRed) + g * 256;
        float* s_mref = reinterpret_cast<float*>(sm + TS::kMref) + g * 64;
        float* s_alpha = reinterpret_cast<float*>(sm + TS::kAlpha) + g * 64;
        float* s_ltot = reinterpret_cast<float*>(sm + TS::kLtot) + g * 64;
        uint8_t* p_buf = sm + TS::kP + g * TS::kPBuf;
        float lsum[NH];
        int n_g = 0;                 // tiles this group has taken
        int p_empty_done = 0;        // this group's PV completions consumed
        long long u_cur = -1, u_done = u_first - 1;
        bool aborted = false;

        auto wait_pv = [&](int upto) {          // PV products of this group's tiles < upto complete
            while (p_empty_done < upto && !aborted) {
                if (!mbar_wait(&bars[kBarPEmpty + g], p_empty_done & 1)) {
                    raise_dev_error(OASIS_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                    aborted = true;
                }
                ++p_empty_done;
            }
        };
        auto partial = [&](long long u) { return NG * (cs + u) + g; };
        // unit end: column sums, then O^T (thread = channel r, its columns)
        // normalised into this group's partial of unit u
        auto finish_unit = [&](long long u) {
            wait_pv(n_g);
            tc_fence_after_sync();
#pragma unroll
            for (int c = 0; c < NH; ++c) {
                float v = lsum[c];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                if (lane == 0) s_red[quad * 64 + cb + c] = v;
            }
            group_bar(g, TS::kGroupThreads);
            if (gt < NQ) s_ltot[gt] = s_red[gt] + s_red[64 + gt] + s_red[128 + gt] + s_red[192 + gt];
            group_bar(g, TS::kGroupThreads);
            const long long p = partial(u);
            float oh[NH], ol[NH];                    // V.P_head and V.P_rest columns
            tmem_ld_x32(tmem + lane_off + o_col + cb, oh);
            tmem_ld_x32(tmem + lane_off + o_col + NQ + cb, ol);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < NH; ++c) {
                const int col = cb + c;
                if (col < rows) {
                    const float L = s_ltot[col];
                    ws_o[(p * rows + col) * kHeadDim + r] = L > 0.f ? (oh[c] + ol[c]) / L : 0.f;
                }
            }
            if (gt < rows) {
                const float L = s_ltot[gt];
                ws_lse[p * rows + gt] = L > 0.f ? (s_mref[gt] + log2f(L)) * kLn2 : kNegInf;
            }
            tc_fence_before_sync();
            group_bar(g, TS::kGroupThreads);
        };
        auto write_empty = [&](long long u) {
            if (gt < rows) ws_lse[partial(u) * rows + gt] = kNegInf;
        };

        // The abort decision is taken from one snapshot after the group
        // barrier, so a group's warps always leave together (a named barrier
        // has no timeout).
        for (int i = 0, t = 0; i < n_list; ++t) {
            const int e = tc_tile_end(l_unit, i, n_list);
            if (NG == 2 && (t & 1) != g) {          // the other group's tile
                i = e;
                continue;
            }
            const long long u = l_unit[i];
            if (u != u_cur) {
                if (u_cur >= 0) {
                    finish_unit(u_cur);
                    u_done = u_cur;
                }
                for (long long uu = u_done + 1; uu < u; ++uu) write_empty(uu);
                u_done = u - 1;
                if (gt < 64) s_mref[gt] = kNegInf;
#pragma unroll
                for (int c = 0; c < NH; ++c) lsum[c] = 0.f;
                u_cur = u;
                group_bar(g, TS::kGroupThreads);
            }
            const int sb = t & 1, vb = t % kVBufs;
            if (!mbar_wait(&bars[kBarSFull + sb], (t >> 1) & 1)) {
                raise_dev_error(OASIS_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            tc_fence_after_sync();
            float x[NH];
            tmem_ld_x32(tmem + lane_off + sb * 64 + cb, x);
            tmem_ld_wait();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kBarSEmpty + sb]);

            const int slot_j = r >> 4, tok = r & 15;
            const bool in_tile = slot_j < e - i;
            const int nv = in_tile ? l_nv[i + slot_j] : 0;
            const bool valid = tok < nv;

            // one group barrier per tile: does any value exceed the reference
            // max by more than 8, and has any role aborted?
            bool need = false;
#pragma unroll
            for (int c = 0; c < NH; ++c)
                if (cb + c < rows && valid && x[c] * scale_log2 > s_mref[cb + c] + 8.f) need = true;
            const unsigned any = __ballot_sync(0xFFFFFFFFu, need);
            const int par = n_g & 1;
            if (lane == 0) s_misc[8 + 8 * par + sw] = any ? 1 : 0;
            if (gt == 0) s_misc[2 + 2 * par + g] = *abort_flag;
            group_bar(g, TS::kGroupThreads);
            if (s_misc[2 + 2 * par + g]) break;
            int rescale = 0;
#pragma unroll
            for (int w = 0; w < kGW; ++w) rescale |= s_misc[8 + 8 * par + gw0 + w];
            if (rescale) {
                // exact column max of this tile, new reference, rescale factors
#pragma unroll
                for (int c = 0; c < NH; ++c) {
                    float v = (valid && cb + c < rows) ? x[c] : kNegInf;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
                    if (lane == 0) s_red[quad * 64 + cb + c] = v;
                }
                group_bar(g, TS::kGroupThreads);
                if (gt < 64) {
                    float a = 1.f;
                    if (gt < rows && gt < NQ) {
                        const float tm =
                            fmaxf(fmaxf(s_red[gt], s_red[64 + gt]), fmaxf(s_red[128 + gt], s_red[192 + gt])) *
                            scale_log2;
                        const float mo = s_mref[gt];
                        if (tm > mo + 8.f) {
                            a = exp2f(mo - tm);          // 0 when mo = -inf
                            s_mref[gt] = tm;
                        }
                    }
                    s_alpha[gt] = a;
                }
                group_bar(g, TS::kGroupThreads);
#pragma unroll
                for (int c = 0; c < NH; ++c) lsum[c] *= s_alpha[cb + c];
                // O^T holds this group's earlier tiles of the unit: scale this
                // thread's channel row for its columns
                wait_pv(n_g);
                tc_fence_after_sync();
#pragma unroll 1
                for (int part = 0; part < 4; ++part) {       // head and rest columns, 16 at a time
                    const int c0 = (part & 1) * 16;
                    const uint32_t col = o_col + (part >> 1) * NQ + cb + c0;
                    uint32_t ov[16];
                    tmem_ld_x16(tmem + lane_off + col, ov);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        ov[c] = __float_as_uint(__uint_as_float(ov[c]) * s_alpha[cb + c0 + c]);
                    tmem_st_x16(tmem + lane_off + col, ov);
                }
                tmem_st_wait();
                tc_fence_before_sync();
            }

            // P^T row r, this thread's columns (head and remainder)
            uint32_t ph[NH / 2], pl[NH / 2];
#pragma unroll
            for (int c2 = 0; c2 < NH / 2; ++c2) {
                float pv[2];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int c = 2 * c2 + k;
                    const float pe = (valid && cb + c < rows) ? exp2f(fmaf(x[c], scale_log2, -s_mref[cb + c])) : 0.f;
                    pv[k] = pe;
                    lsum[c] += pe;
                }
                ph[c2] = pack_bf16x2(pv[0], pv[1]);
                pl[c2] = pack_bf16x2(pv[0] - bf16_lo(ph[c2]), pv[1] - bf16_hi(ph[c2]));
            }
            wait_pv(n_g);                                   // this group's previous PV read P
            // P^T row r: columns [0, NQ) hold the bf16 head, [NQ, 2NQ) the
            // remainder; 64 columns per 128-B swizzled atom of 128 rows
            uint8_t* prow = p_buf + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
            for (int k = 0; k < NH / 8; ++k) {
                const int ch = cb / 8 + k, cl = (NQ + cb) / 8 + k;
                *reinterpret_cast<uint4*>(prow + (ch >> 3) * kTcRegion + (((ch & 7) ^ (r & 7)) << 4)) =
                    make_uint4(ph[4 * k], ph[4 * k + 1], ph[4 * k + 2], ph[4 * k + 3]);
                *reinterpret_cast<uint4*>(prow + (cl >> 3) * kTcRegion + (((cl & 7) ^ (r & 7)) << 4)) =
                    make_uint4(pl[4 * k], pl[4 * k + 1], pl[4 * k + 2], pl[4 * k + 3]);
            }
            // masked tokens of a loaded block: zero their V row once it has
            // landed (it may hold anything beyond the context)
            if (in_tile && !valid) {
                if (!mbar_wait(&bars[kBarVFull + vb], (t / kVBufs) & 1)) {
                    raise_dev_error(OASIS_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                }
                uint8_t* vrow = sm + TS::kV + vb * kTcHalfBytes + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                for (int reg = 0; reg < 2; ++reg) {
                    if (TS::kHalves == 2 && reg != half) continue;   // two column halves split the regions
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        *reinterpret_cast<uint4*>(vrow + reg * kTcRegion + ch * 16) = make_uint4(0, 0, 0, 0);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kBarPFull + g]);
            ++n_g;
            i = e;
        }
        if (gt == 0) s_misc[6 + g] = *abort_flag;
        group_bar(g, TS::kGroupThreads);
        if (u_cur >= 0 && !s_misc[6 + g]) {
            finish_unit(u_cur);
            u_done = u_cur;
        }
        for (long long uu = u_done + 1; uu <= u_last; ++uu) write_empty(uu);
    }
    tc_fence_before_sync();
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == 1) tmem_dealloc(tmem, kTcTmemCols);
}

}  // namespace oasis
