// attn.cuh - sparse GQA decode attention over the resident pool slots.
//
// OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
// Prefetching, Figure 7 (right): the verification query and the drafts are
// attended in one pass over the resident sparse working set; Figure 9: the
// per-head slot table says which block each pool slot holds.
//
// Work split (stream-K): the T = B*Hkv*K pool slots, in (sequence, KV head,
// slot) order, are cut into NS contiguous ranges, one per "stream".  A
// stream is QG warps that share a 3-stage ring of 8 KiB shared-memory
// buffers; its first warp's lane 0 fills the ring with TMA (two 64-column
// boxes per slot, 128-byte swizzle, L2 evict-first), skipping free slots and
// blocks beyond the context.  Streams are independent - there is no CTA-wide
// barrier anywhere in the kernel - so an SM keeps up to 8 streams x 24 KiB
// of KV in flight.  A stream writes one normalised partial (output and
// log-sum-exp) for every (sequence, KV head) unit its range touches; a second
// kernel, launched as a programmatic dependent, merges the partials of each
// unit in stream order (one warp per query row, every load in flight).
//
// Math per slot (16 tokens), per warp, on the warp-level tensor-core path
// (mma.sync m16n8k16, bf16 in, fp32 accumulate), tokens as the M dimension
// and the Qn*G query rows of the KV head as N (8 per n-tile):
//   S^T[16 x 8] = K[16 x 128] . Q^T           (8 k-steps per n-tile)
//   online softmax per query column (max over tokens by xor-shuffles)
//   P^T fragments -> PV B operand by movmatrix.trans (no smem round trip);
//   P enters as a bf16 head plus a bf16 remainder (two MMAs), so the weights
//   keep ~16 significant bits
//   O^T[128 x 8] += V^T[128 x 16] . P^T       (8 m-tiles per n-tile)
// With more than 4 n-tiles (Qn*G > 32) a stream is two warps, each owning
// half of the query n-tiles.
#pragma once

#include "common.cuh"

namespace oasis {

constexpr int kAttnStreamsPerCta = 4;
constexpr int kAttnStages = 3;
constexpr int kAttnWindow = 256;                          // slots listed per pass
constexpr int kAttnStreamSmem = kAttnStages * kBlockBytes + kAttnWindow * 8 + 64;
constexpr float kLn2 = 0.6931471805599453f;

template <int NTW, int QG>
struct AttnCfg {
    static constexpr int kWarps = kAttnStreamsPerCta * QG;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kStreamStride = (kAttnStreamSmem + 1023) / 1024 * 1024;
    static constexpr int kSmem = kAttnStreamsPerCta * kStreamStride + 1024;
};

// Streams whose ranges touch unit u: [first, last].  Slot s belongs to
// stream floor(s * NS / T), so every stream in between touches u.
__host__ __device__ __forceinline__ void attn_unit_streams(long long u, long long K, long long NS, long long T,
                                                           long long* first, long long* last) {
    *first = (u * K) * NS / T;
    *last = ((u + 1) * K - 1) * NS / T;
}

// floor(x / t) for x < 2^53, t < 2^31 without the 64-bit integer division
// routine: a double quotient, then an exact integer correction.
__device__ __forceinline__ long long floor_div_small(long long x, long long t) {
    long long q = static_cast<long long>(static_cast<double>(x) / static_cast<double>(t));
    if (q * t > x) --q;
    else if ((q + 1) * t <= x) ++q;
    return q;
}

// Merges the stream partials of each (unit, query row) in stream order:
// lse = log sum_p exp(lse_p), out = sum_p exp(lse_p - lse) * o_p.  One warp
// per (unit, row); lane j holds partial j's lse, lane c owns channels
// 4c..4c+3.  Up to 12 partials (the usual case: 8 streams per SM give about
// 10 per unit on the 32K Llama layer) are read in one round trip: every lse
// and output load is issued before any of them is used.  Small CTAs, and at
// most 80 registers so that 12 CTAs fit an SM and the grid runs in one wave.
constexpr int kMergeWarps = 2;
constexpr int kMergeFast = 12;

__global__ void __launch_bounds__(32 * kMergeWarps, 12) attn_merge_kernel(Dims d, int n_streams,
                                                                      const float* __restrict__ ws_o,
                                                                      const float* __restrict__ ws_lse,
                                                                      float* __restrict__ out,
                                                                      float* __restrict__ lse_out) {
    const float kNegInf = -__int_as_float(0x7f800000);
    const int lane = threadIdx.x & 31;
    const int G = d.G();
    const int rows = d.Qn * G;
    const int units = d.B * d.Hkv;
    const int gw = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);   // < units * rows <= 2^22
    // partials are produced by the attention grid this kernel depends on
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (gw >= units * rows) return;
    const int u = gw / rows;
    const int r = gw - u * rows;
    // streams whose ranges touch unit u (attn_unit_streams): slot s is in stream floor(s*NS/T)
    const long long T = static_cast<long long>(units) * d.K;
    const long long first = floor_div_small(static_cast<long long>(u) * d.K * n_streams, T);
    const long long last = floor_div_small((static_cast<long long>(u + 1) * d.K - 1) * n_streams, T);
    const int np = static_cast<int>(last - first + 1);
    const long long p0 = first + u;
    const float4* src = reinterpret_cast<const float4*>(ws_o + (p0 * rows + r) * kHeadDim) + lane;
    const long long pstride = static_cast<long long>(rows) * (kHeadDim / 4);
    float M = kNegInf, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (np <= kMergeFast) {
        const float lj = lane < np ? ws_lse[(p0 + lane) * rows + r] : kNegInf;
        float4 v[kMergeFast];
#pragma unroll
        for (int k = 0; k < kMergeFast; ++k) v[k] = k < np ? src[k * pstride] : make_float4(0.f, 0.f, 0.f, 0.f);
        M = lj;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
        const float wj = (lj == kNegInf) ? 0.f : __expf(lj - M);
        L = wj;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xFFFFFFFFu, L, o);
#pragma unroll
        for (int k = 0; k < kMergeFast; ++k) {
            const float w = __shfl_sync(0xFFFFFFFFu, wj, k);
            if (w > 0.f) {                      // empty partials may hold stale outputs
                acc.x += w * v[k].x;
                acc.y += w * v[k].y;
                acc.z += w * v[k].z;
                acc.w += w * v[k].w;
            }
        }
    } else {
        for (int j0 = 0; j0 < np; j0 += 32) {
            const float lj = j0 + lane < np ? ws_lse[(p0 + j0 + lane) * rows + r] : kNegInf;
            M = fmaxf(M, lj);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
        if (M != kNegInf) {
            for (int j0 = 0; j0 < np; j0 += 32) {
                const float lj = j0 + lane < np ? ws_lse[(p0 + j0 + lane) * rows + r] : kNegInf;
                const float wj = lj == kNegInf ? 0.f : __expf(lj - M);
                float ws = wj;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ws += __shfl_xor_sync(0xFFFFFFFFu, ws, o);
                L += ws;
                const int nj = min(32, np - j0);
                for (int k0 = 0; k0 < nj; k0 += 8) {
                    float4 v[8];
                    float wk[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        wk[k] = __shfl_sync(0xFFFFFFFFu, wj, (k0 + k) & 31);
                        v[k] = (k0 + k < nj && wk[k] > 0.f) ? src[(j0 + k0 + k) * pstride]
                                                            : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float w = k0 + k < nj ? wk[k] : 0.f;
                        acc.x += w * v[k].x;
                        acc.y += w * v[k].y;
                        acc.z += w * v[k].z;
                        acc.w += w * v[k].w;
                    }
                }
            }
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
    const int b = u / d.Hkv, h = u - b * d.Hkv;
    const long long orow = (static_cast<long long>(b) * d.Qn + r / G) * d.Hq + h * G + r % G;
    reinterpret_cast<float4*>(out + orow * kHeadDim)[lane] = acc;
    if (lane == 0) lse_out[orow] = L > 0.f ? M + logf(L) : kNegInf;
}

template <int NTW, int QG>
__global__ void __launch_bounds__(AttnCfg<NTW, QG>::kThreads)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_pool, Dims d, const uint16_t* __restrict__ q,
                       const int32_t* __restrict__ slot_table, const int32_t* __restrict__ ctx_len,
                       float scale_log2, int n_streams, float* __restrict__ ws_o, float* __restrict__ ws_lse) {
    using Cfg = AttnCfg<NTW, QG>;
    const float kNegInf = -__int_as_float(0x7f800000);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ls = warp / QG, qg = warp % QG;             // local stream, query group
    const long long gs = static_cast<long long>(blockIdx.x) * kAttnStreamsPerCta + ls;

    uint8_t* ring = smem + ls * Cfg::kStreamStride;
    int* l_slot = reinterpret_cast<int*>(ring + kAttnStages * kBlockBytes);
    int* l_nv = l_slot + kAttnWindow;
    uint64_t* full = reinterpret_cast<uint64_t*>(l_nv + kAttnWindow);   // [stages]
    uint64_t* empty = full + kAttnStages;                                // [stages]

    const int g = lane >> 2, t = lane & 3;
    const int G = d.G();
    const int rows = d.Qn * G;
    const long long K = d.K;
    const long long T = static_cast<long long>(d.B) * d.Hkv * K;
    const long long s_begin = gs < n_streams ? (gs * T + n_streams - 1) / n_streams : 0;
    const long long s_end = gs < n_streams ? ((gs + 1) * T + n_streams - 1) / n_streams : 0;
    const long long u_first = s_begin / K, u_last = (s_end - 1) / K;
    if (s_begin < s_end) {

    if (qg == 0) {
        if (lane < kAttnStages) {
            mbar_init(&full[lane], 1);
            mbar_init(&empty[lane], QG);
        }
        fence_mbar_init();
    }
    if (QG > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + ls), "r"(32 * QG) : "memory");
    __syncwarp();

    const uint64_t pol = l2_policy_evict_first();
    const uint32_t ring_addr = smem_addr(ring);
    auto issue = [&](int idx, long long pos) {
        const int stage = static_cast<int>(pos % kAttnStages);
        uint64_t* bar = &full[stage];
        const int y = l_slot[idx] * (2 * kBlockTokens);
        mbar_arrive_expect_tx(bar, kBlockBytes);
        tma_load_2d(ring + stage * kBlockBytes, &tm_pool, bar, 0, y, pol);
        tma_load_2d(ring + stage * kBlockBytes + kBlockBytes / 2, &tm_pool, bar, 64, y, pol);
    };

    float o[8][NTW][4];
    float m_run[NTW][2], l_run[NTW][2];
    uint32_t qf[NTW][8][2];

    auto load_unit = [&](long long u) {
        const int b = static_cast<int>(u / d.Hkv), h = static_cast<int>(u % d.Hkv);
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt) {
            const int r = 8 * (qg * NTW + nt) + g;
            const bool valid = r < rows;
            const uint16_t* qrow = q + ((static_cast<long long>(b) * d.Qn + (valid ? r / G : 0)) * d.Hq + h * G +
                                        (valid ? r % G : 0)) *
                                           kHeadDim;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                qf[nt][ks][0] = valid ? __ldg(reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * t)) : 0u;
                qf[nt][ks][1] = valid ? __ldg(reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * t + 8)) : 0u;
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                m_run[nt][c] = kNegInf;
                l_run[nt][c] = 0.f;
            }
#pragma unroll
            for (int mt = 0; mt < 8; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) o[mt][nt][e] = 0.f;
        }
    };

    // Normalised partial of unit u into entry p = gs + u of the workspace
    // (unique: a later stream starts at or after this stream's last unit).
    auto finalize = [&](long long u, bool any) {
        const long long p = gs + u;
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float l = l_run[nt][c];
                l += __shfl_xor_sync(0xFFFFFFFFu, l, 4);
                l += __shfl_xor_sync(0xFFFFFFFFu, l, 8);
                l += __shfl_xor_sync(0xFFFFFFFFu, l, 16);
                const int col = 8 * (qg * NTW + nt) + 2 * t + c;
                const bool live = any && l > 0.f;
                const float inv = live ? 1.f / l : 0.f;
                if (col < rows) {
                    if (g == 0) ws_lse[p * rows + col] = live ? (m_run[nt][c] + log2f(l)) * kLn2 : kNegInf;
                    if (live) {
                        float* dst = ws_o + (p * rows + col) * kHeadDim;
#pragma unroll
                        for (int mt = 0; mt < 8; ++mt) {
                            dst[16 * mt + g] = o[mt][nt][c] * inv;
                            dst[16 * mt + g + 8] = o[mt][nt][2 + c] * inv;
                        }
                    }
                }
            }
        }
    };
    auto write_empty = [&](long long u) {
        const long long p = gs + u;
        const int c1 = min(rows, 8 * (qg + 1) * NTW);
        for (int col = 8 * qg * NTW + lane; col < c1; col += 32) ws_lse[p * rows + col] = kNegInf;
    };

    const int rowK = lane & 15, hiK = lane >> 4;
    const int tokV = (lane & 7) + ((lane >> 4) << 3), hiV = (lane >> 3) & 1;
    long long rp = 0;            // ring position of the next slot consumed
    long long u_cur = -1;
    long long u_end = 0;         // first slot past the current unit
    bool any = false;            // the current unit has seen a slot
    bool failed = false;

    // A failed (timed-out) wait does not leave the loops early: every warp of
    // a stream must reach the same named barriers, so the remaining slots are
    // walked without waiting or computing.
    for (long long w0 = s_begin; w0 < s_end; w0 += kAttnWindow) {
        const long long w1 = min(s_end, w0 + kAttnWindow);
        // ---- the occupied slots of this window, in slot order
        int n_list = 0;
        for (long long base = w0; base < w1; base += 32) {
            const long long s = base + lane;
            int nv = 0;
            if (s < w1) {
                int blk = slot_table[s];
                if (blk < -1 || blk >= d.N) {
                    if (qg == 0) raise_dev_error(OASIS_DEVERR_ID_RANGE);
                    blk = -1;
                }
                // slot indices stay below 2^26 (host check): 32-bit division
                const unsigned unit = static_cast<unsigned>(s) / static_cast<unsigned>(K);
                if (blk >= 0) nv = min(kBlockTokens, ctx_len[unit / static_cast<unsigned>(d.Hkv)] - blk * kBlockTokens);
            }
            const unsigned m = __ballot_sync(0xFFFFFFFFu, nv > 0);
            if (nv > 0 && qg == 0) {
                const int pos = n_list + __popc(m & ((1u << lane) - 1u));
                l_slot[pos] = static_cast<int>(s);
                l_nv[pos] = nv;
            }
            n_list += __popc(m);
        }
        if (QG > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + ls), "r"(32 * QG) : "memory");
        __syncwarp();
        if (qg == 0 && lane == 0 && !failed)
            for (int i = 0; i < kAttnStages && i < n_list; ++i) issue(i, rp + i);

        for (int i = 0; i < n_list; ++i, ++rp) {
            if (l_slot[i] >= u_end) {
                // slots are listed in order: divide only when the unit changes
                const long long u = l_slot[i] / K;
                if (u_cur >= 0) finalize(u_cur, any);
                for (long long uu = (u_cur < 0 ? u_first : u_cur + 1); uu < u; ++uu) write_empty(uu);
                u_cur = u;
                u_end = (u + 1) * K;
                any = false;
                load_unit(u);
            }
            if (failed) continue;
            const int stage = static_cast<int>(rp % kAttnStages);
            const uint32_t parity = static_cast<uint32_t>((rp / kAttnStages) & 1);
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[stage], parity))) {
                if (lane == 0) raise_dev_error(OASIS_DEVERR_TIMEOUT);
                failed = true;
                continue;
            }
            any = true;
            const int nv = l_nv[i];
            const uint32_t sbase = ring_addr + stage * kBlockBytes;

            // S^T = K . Q^T
            float sacc[NTW][4];
#pragma unroll
            for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int c16 = ((ks & 3) << 1) | hiK;
                const uint32_t addr = sbase + (ks >> 2) * (kBlockBytes / 2) + rowK * 128 + ((c16 ^ (rowK & 7)) << 4);
                uint32_t a[4];
                ldsm_x4(addr, a);
#pragma unroll
                for (int nt = 0; nt < NTW; ++nt) mma_bf16_m16n8k16(sacc[nt], a, qf[nt][ks][0], qf[nt][ks][1]);
            }
            if (nv < kBlockTokens) {
#pragma unroll
                for (int nt = 0; nt < NTW; ++nt) {
                    if (g >= nv) sacc[nt][0] = sacc[nt][1] = kNegInf;
                    if (g + 8 >= nv) sacc[nt][2] = sacc[nt][3] = kNegInf;
                }
            }
            // online softmax over tokens, per query column (log2 domain).  The
            // reference max only moves when a tile's max exceeds it by more
            // than 8 (weights stay <= 2^8), so O and l are rarely rescaled;
            // lse = m + log2(l) is exact for any reference.  scale > 0.
            float alpha[NTW][2];
            bool rescale = false;
#pragma unroll
            for (int nt = 0; nt < NTW; ++nt) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float mx = fmaxf(sacc[nt][c], sacc[nt][2 + c]);
                    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 16));
                    const float mx_s = mx * scale_log2;
                    alpha[nt][c] = 1.f;
                    if (mx_s > m_run[nt][c] + 8.f) {
                        alpha[nt][c] = exp2f(m_run[nt][c] - mx_s);
                        m_run[nt][c] = mx_s;
                        rescale = true;
                    }
                    sacc[nt][c] = exp2f(fmaf(sacc[nt][c], scale_log2, -m_run[nt][c]));
                    sacc[nt][2 + c] = exp2f(fmaf(sacc[nt][2 + c], scale_log2, -m_run[nt][c]));
                }
            }
            if (__any_sync(0xFFFFFFFFu, rescale)) {
#pragma unroll
                for (int nt = 0; nt < NTW; ++nt) {
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        o[mt][nt][0] *= alpha[nt][0];
                        o[mt][nt][1] *= alpha[nt][1];
                        o[mt][nt][2] *= alpha[nt][0];
                        o[mt][nt][3] *= alpha[nt][1];
                    }
                    l_run[nt][0] *= alpha[nt][0];
                    l_run[nt][1] *= alpha[nt][1];
                }
            }
            // P^T -> B fragments of O^T += V^T . P^T (head + remainder)
            uint32_t pb[NTW][2], pr[NTW][2];
#pragma unroll
            for (int nt = 0; nt < NTW; ++nt) {
                const uint32_t h0 = pack_bf16x2(sacc[nt][0], sacc[nt][1]);   // token g
                const uint32_t h1 = pack_bf16x2(sacc[nt][2], sacc[nt][3]);   // token g + 8
                const uint32_t r0 = pack_bf16x2(sacc[nt][0] - bf16_lo(h0), sacc[nt][1] - bf16_hi(h0));
                const uint32_t r1 = pack_bf16x2(sacc[nt][2] - bf16_lo(h1), sacc[nt][3] - bf16_hi(h1));
                l_run[nt][0] += sacc[nt][0] + sacc[nt][2];
                l_run[nt][1] += sacc[nt][1] + sacc[nt][3];
                pb[nt][0] = movmatrix_trans(h0);
                pb[nt][1] = movmatrix_trans(h1);
                pr[nt][0] = movmatrix_trans(r0);
                pr[nt][1] = movmatrix_trans(r1);
            }
            uint32_t vmask_lo = 0xFFFFFFFFu, vmask_hi = 0xFFFFFFFFu;
            if (nv < kBlockTokens) {
                vmask_lo = (2 * t < nv ? 0xFFFFu : 0u) | (2 * t + 1 < nv ? 0xFFFF0000u : 0u);
                vmask_hi = (2 * t + 8 < nv ? 0xFFFFu : 0u) | (2 * t + 9 < nv ? 0xFFFF0000u : 0u);
            }
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const int row = kBlockTokens + tokV;
                const int c16 = ((mt & 3) << 1) | hiV;
                const uint32_t addr = sbase + (mt >> 2) * (kBlockBytes / 2) + row * 128 + ((c16 ^ (row & 7)) << 4);
                uint32_t a[4];
                ldsm_x4_trans(addr, a);
                a[0] &= vmask_lo;
                a[1] &= vmask_lo;
                a[2] &= vmask_hi;
                a[3] &= vmask_hi;
#pragma unroll
                for (int nt = 0; nt < NTW; ++nt) {
                    mma_bf16_m16n8k16(o[mt][nt], a, pb[nt][0], pb[nt][1]);
                    mma_bf16_m16n8k16(o[mt][nt], a, pr[nt][0], pr[nt][1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (qg == 0 && lane == 0 && i + kAttnStages < n_list) {
                if (mbar_wait(&empty[stage], parity)) {
                    fence_proxy_async_smem();
                    issue(i + kAttnStages, rp + kAttnStages);
                } else {
                    raise_dev_error(OASIS_DEVERR_TIMEOUT);
                    failed = true;
                }
            }
            __syncwarp();
        }
        // every warp of the stream is done with this window's list
        if (QG > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + ls), "r"(32 * QG) : "memory");
    }
    if (u_cur >= 0) finalize(u_cur, any);
    for (long long uu = (u_cur < 0 ? u_first : u_cur + 1); uu <= u_last; ++uu) write_empty(uu);
    }   // s_begin < s_end
    // let the merge kernel (launched as a programmatic dependent) start early
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace oasis
