// oasis.cu - C ABI of the lookahead sparse-KV decode path (see include/oasis.h).
//
// Host side: argument validation before anything is enqueued, TMA tensor-map
// encoding, workspace layout and kernel launches.  All kernels live in the
// .cuh files included below so the library is one translation unit (the
// device error word needs no relocatable device code).

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <mutex>

#include "oasis.h"

#include "attn.cuh"
#include "common.cuh"
#include "fused.cuh"
#include "overlap.cuh"
#include "plan.cuh"
#include "prefetch.cuh"
#include "score.cuh"
#include "select.cuh"
#include "summaries.cuh"

namespace {

using oasis::Dims;

thread_local char g_msg[512] = "";

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(OASIS_ECUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

int check_launch(const char* what) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, what);
    g_msg[0] = '\0';
    return OASIS_OK;
}

int validate(const oasis_dims* dp, Dims* out) {
    if (dp == nullptr) return fail(OASIS_EINVAL, "dims is NULL");
    const oasis_dims& d = *dp;
    if (d.head_dim != oasis::kHeadDim) return fail(OASIS_EINVAL, "head_dim must be 128 (got %d)", d.head_dim);
    if (d.block_tokens != oasis::kBlockTokens)
        return fail(OASIS_EINVAL, "block_tokens must be 16 (got %d)", d.block_tokens);
    if (d.batch < 1 || d.n_kv_heads < 1 || d.n_q_heads < 1)
        return fail(OASIS_EINVAL, "batch, n_q_heads and n_kv_heads must be >= 1");
    if (d.n_q_heads % d.n_kv_heads != 0)
        return fail(OASIS_EINVAL, "n_q_heads (%d) must be a multiple of n_kv_heads (%d)", d.n_q_heads, d.n_kv_heads);
    if (d.budget_blocks < 1 || d.budget_blocks > 1024)
        return fail(OASIS_EINVAL, "budget_blocks must be in [1, 1024] (got %d)", d.budget_blocks);
    if (d.max_blocks < d.budget_blocks || d.max_blocks > 32768)
        return fail(OASIS_EINVAL, "max_blocks must be in [budget_blocks, 32768] (got %d)", d.max_blocks);
    if (d.fetch_cap < 0 || d.fetch_cap > d.budget_blocks)
        return fail(OASIS_EINVAL, "fetch_cap must be in [0, budget_blocks] (got %d)", d.fetch_cap);
    if (d.n_queries < 1) return fail(OASIS_EINVAL, "n_queries must be >= 1");
    const int G = d.n_q_heads / d.n_kv_heads;
    if (static_cast<long long>(d.n_queries) * G > 64)
        return fail(OASIS_EINVAL, "n_queries * G must be <= 64 (got %d)", d.n_queries * G);
    const long long units = static_cast<long long>(d.batch) * d.n_kv_heads;
    if (units > 65535) return fail(OASIS_EINVAL, "batch * n_kv_heads must be <= 65535");
    if (units * d.max_blocks * 32 > 0x7FFFFFFFll || units * d.budget_blocks * 32 > 0x7FFFFFFFll)
        return fail(OASIS_EINVAL, "tensor too large for 32-bit row coordinates");
    if (out) *out = Dims{d.batch, d.n_q_heads, d.n_kv_heads, d.head_dim, d.block_tokens,
                         d.max_blocks, d.budget_blocks, d.n_queries, d.fetch_cap};
    return OASIS_OK;
}

int check_ptr(const void* p, const char* name, bool nullable = false) {
    if (p == nullptr) return nullable ? OASIS_OK : fail(OASIS_EINVAL, "%s is NULL", name);
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return fail(OASIS_EINVAL, "%s is not 16-byte aligned", name);
    return OASIS_OK;
}

// Resolves a pointer the device may read: device memory as is, pinned host
// memory through its device mapping.  `allow_device` rejects device memory
// when only mapped host memory makes sense.
int device_view(const void* p, const char* name, bool allow_device, const void** out) {
    cudaPointerAttributes a;
    const cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(OASIS_ENOTMAPPED, "%s: cudaPointerGetAttributes failed (%s)", name, cudaGetErrorName(e));
    }
    if (a.type == cudaMemoryTypeHost) {
        if (a.devicePointer == nullptr) return fail(OASIS_ENOTMAPPED, "%s: pinned host memory is not mapped", name);
        *out = a.devicePointer;
        return OASIS_OK;
    }
    if ((a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) && allow_device) {
        *out = p;
        return OASIS_OK;
    }
    return fail(OASIS_ENOTMAPPED, "%s: not %s", name, allow_device ? "device or mapped pinned host memory"
                                                                   : "mapped pinned host memory");
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        cudaGetLastError();
    });
    return fn;
}

// bf16 matrix [rows][128] with 256-B rows, boxes of 64 columns x box_rows,
// 128-byte swizzle.
int make_map(CUtensorMap* m, const void* base, unsigned long long rows, unsigned box_rows, const char* name) {
    auto fn = encode_fn();
    if (fn == nullptr) return fail(OASIS_ECUDA, "cuTensorMapEncodeTiled unavailable");
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(oasis::kHeadDim), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(oasis::kRowBytes)};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(OASIS_ECUDA, "cuTensorMapEncodeTiled(%s) failed: %d", name, static_cast<int>(r));
    return OASIS_OK;
}

// Keys (or values, from base + 4 KiB) of the pool: bf16 [B*Hkv*K slots][32
// rows][128] seen as a 3-D tensor (128 columns, 16 rows of one slot's K or V,
// slots 8 KiB apart), boxes of 64 columns x 16 rows x 4 consecutive slots.
int make_map_pool(CUtensorMap* m, const void* base, unsigned long long slots, const char* name) {
    auto fn = encode_fn();
    if (fn == nullptr) return fail(OASIS_ECUDA, "cuTensorMapEncodeTiled unavailable");
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(oasis::kHeadDim), static_cast<cuuint64_t>(oasis::kBlockTokens),
                                static_cast<cuuint64_t>(slots)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(oasis::kRowBytes),
                                   static_cast<cuuint64_t>(oasis::kBlockBytes)};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(oasis::kBlockTokens),
                               static_cast<cuuint32_t>(oasis::kAttnTileSlots)};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(OASIS_ECUDA, "cuTensorMapEncodeTiled(%s) failed: %d", name, static_cast<int>(r));
    return OASIS_OK;
}

// The query rows of every (sequence, KV head): bf16 q [B][Qn][Hq][128] seen
// as a 3-D tensor (128 columns, Hq heads, B*Qn query positions), boxes of
// 64 columns x G heads x nq positions, so one box per 64-column half brings
// nq of the unit's query positions in (j, g) order, 128-byte swizzled.
int make_map_q(CUtensorMap* m, const void* q, const Dims& d, int nq) {
    auto fn = encode_fn();
    if (fn == nullptr) return fail(OASIS_ECUDA, "cuTensorMapEncodeTiled unavailable");
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(oasis::kHeadDim), static_cast<cuuint64_t>(d.Hq),
                                static_cast<cuuint64_t>(d.B) * d.Qn};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(oasis::kRowBytes),
                                   static_cast<cuuint64_t>(oasis::kRowBytes) * d.Hq};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(d.G()), static_cast<cuuint32_t>(nq)};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(OASIS_ECUDA, "cuTensorMapEncodeTiled(q) failed: %d", static_cast<int>(r));
    return OASIS_OK;
}

// Every kernel asks for the largest shared-memory carve-out.  An SM's split
// between L1 and shared memory is set when a CTA lands on an idle SM, and an
// SM split for a kernel that needs little shared memory (the gather, the
// plan) cannot take a 200-KB attention or scoring CTA until it drains: the
// attention launched beside a running gather then ran in two waves.
template <typename K>
int carveout(K kernel, const char* what) {
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return cuda_fail(e, what);
    return OASIS_OK;
}

template <typename K>
int set_smem(K kernel, int bytes, const char* what) {
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return cuda_fail(e, what);
    return carveout(kernel, what);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Attention chunks: a unit's ceil(K / 8) tiles cut into chunks of `ct`
// tiles.  Every chunk costs a running-max seed, a pipeline refill and, for a
// split unit, a partial write and its share of the merge; on B200 whole-unit
// chunks were fastest when there are about as many units as SMs (a 32K layer
// of 128 units: 38.9 us whole against 43.0 / 51.2 / 65.7 us for 8 / 4 / 2
// tiles per chunk).  So units are split only when there are fewer of them
// than CTAs, into about CTAs / units chunks; chunks are at least 2 tiles (4
// with more than 32 query rows) so a split unit's partials stay under ~1/8 of
// the bytes it reads, and a unit has at most 8 of them (the merge's limit).
int attn_min_chunk_tiles(const Dims& d) {
    const int tpu = (d.K + oasis::kAttnTileSlots - 1) / oasis::kAttnTileSlots;
    return std::min(tpu, d.Qn * d.G() <= 32 ? 2 : 4);
}

oasis::AttnChunks attn_chunks(const Dims& d, int ctas) {
    const int tpu = (d.K + oasis::kAttnTileSlots - 1) / oasis::kAttnTileSlots;
    const long long units = static_cast<long long>(d.B) * d.Hkv;
    const int want = static_cast<int>(std::max<long long>(1, ctas / std::max(1ll, units)));   // chunks a unit
    int ct = (tpu + want - 1) / want;
    ct = std::max(ct, attn_min_chunk_tiles(d));
    ct = std::min(ct, oasis::kAttnMaxChunkTiles);
    ct = std::max(ct, (tpu + oasis::kAttnMaxChunks - 1) / oasis::kAttnMaxChunks);   // the merge takes <= 8
    ct = std::min(ct, tpu);
    oasis::AttnChunks c;
    c.ct = ct;
    c.cpu = (tpu + ct - 1) / ct;
    c.nc = static_cast<int>(units * c.cpu);
    return c;
}

// Workspace: block scores [B*Hkv*N] fp32, then the attention partials of
// split units (log2-sum-exp [P][rows] and normalised outputs [P][rows][128],
// P = the most chunks any launch makes), then one ticket counter per unit
// for the attention merge, one per unit for the fused score / select / plan,
// the attention's chunk and exit counters and the fused scoring's chunk,
// exit and tail-claim counters (all zero between calls).
struct WsLayout {
    size_t scores, lse, o, ticket, sticket, sched, ssched, total;
    long long partials;
};

WsLayout ws_layout(const Dims& d) {
    WsLayout w;
    const size_t units = static_cast<size_t>(d.B) * d.Hkv;
    const size_t rows = static_cast<size_t>(d.Qn) * d.G();
    const long long tpu = (d.K + oasis::kAttnTileSlots - 1) / oasis::kAttnTileSlots;
    const long long mct = attn_min_chunk_tiles(d);
    w.partials = static_cast<long long>(units) * ((tpu + mct - 1) / mct);
    w.scores = 0;
    w.lse = align256(units * d.N * sizeof(float));
    w.o = align256(w.lse + static_cast<size_t>(w.partials) * rows * sizeof(float));
    w.ticket = align256(w.o + static_cast<size_t>(w.partials) * rows * oasis::kHeadDim * sizeof(float));
    w.sticket = align256(w.ticket + units * sizeof(int));
    w.sched = align256(w.sticket + units * sizeof(int));
    w.ssched = align256(w.sched + 2 * sizeof(int));
    w.total = align256(w.ssched + 4 * sizeof(int));
    return w;
}

int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) ==
                                                      cudaSuccess)
            n = v;
        else
            n = 148;
    }
    return n;
}

template <int NPAD>
int launch_score(const CUtensorMap& tmax, const CUtensorMap& tmin, const Dims& d, const uint16_t* q,
                 const int32_t* ctx, float* scores, int row0, int rows, cudaStream_t s) {
    using S = oasis::ScoreSmem<NPAD>;
    auto k = oasis::lookahead_score_kernel<NPAD>;
    if (int rc = set_smem(k, S::kBytes, "score smem")) return rc;
    dim3 grid((d.N + oasis::kScoreTile - 1) / oasis::kScoreTile, d.B * d.Hkv);
    k<<<grid, 128, S::kBytes, s>>>(tmax, tmin, d, q, ctx, scores, row0, rows);
    return check_launch("lookahead_score launch");
}

// Scoring chunks: like the attention's, whole units when there are about as
// many units as SMs (a 32K layer of 128 units: 55.4 us against 59.4 / 61.5 /
// 64.5 / 71.8 us for chunks of 8 / 4 / 2 / 1 tiles of 128 blocks), else about
// CTAs / units chunks a unit.
template <int NPAD, bool kScored>
int launch_fused(const CUtensorMap& tmax, const CUtensorMap& tmin, const CUtensorMap& tq, const Dims& d,
                 const uint16_t* q,
                 const int32_t* ctx, float* scores, int row0, int rows, int* ticket, int* sched, int32_t* sel,
                 float* sel_score, int32_t* st, int32_t* lu, int32_t step, const int32_t* step_dev, int32_t* fs,
                 int32_t* fb, int32_t* nf, cudaStream_t s) {
    using S = oasis::SspSmem<NPAD>;
    auto k = oasis::score_select_plan_kernel<NPAD, kScored>;
    // two unit operands when they fit beside the ring and the tail scratch, else one
    const int nbuf = S::bytes(2, d.K, d.N) <= 227 * 1024 ? 2 : 1;
    const int smem = S::bytes(nbuf, d.K, d.N);
    if (smem > 227 * 1024)
        return fail(OASIS_EINVAL, "budget_blocks %d / max_blocks %d need more shared memory than a CTA has", d.K, d.N);
    if (int rc = set_smem(k, smem, "score_select_plan smem")) return rc;
    const int tpu = (d.N + oasis::kScoreTile - 1) / oasis::kScoreTile;
    oasis::SspChunks ch;
    const long long units = static_cast<long long>(d.B) * d.Hkv;
    // Whole units when there are at least half as many units as SMs (the
    // epilogue hands the keys over in shared memory; cutting units would not
    // shorten the longest CTA's share by more than the hand-off saves).
    // Fewer units: about two chunks per SM (a power of two per unit, at least
    // two tiles a chunk), so every SM scores and the units finish one after
    // another, their selections overlapping the scoring of later units.
    int want = 1;
    if (2 * units < sm_count()) {
        const long long per = (2ll * sm_count() + units - 1) / units;
        while (want < per) want <<= 1;
        want = std::max(1, std::min(want, tpu / 2));
    }
    ch.cts = (tpu + want - 1) / want;
    ch.cpu = (tpu + ch.cts - 1) / ch.cts;
    ch.nc = static_cast<int>(units * ch.cpu);
    ch.whole = ch.cpu == 1 ? 1 : 0;
    const int ctas = std::min(sm_count(), ch.nc);
    k<<<ctas, oasis::kSspThreads, smem, s>>>(tmax, tmin, tq, d, q, ctx, scores, row0, rows, ticket, sched, sel, sel_score,
                                             st, lu, step, step_dev, fs, fb, nf, ch, nbuf);
    return check_launch("score_select_plan launch");
}

template <bool kScored>
int launch_fused_rows(const CUtensorMap& tmax, const CUtensorMap& tmin, const CUtensorMap& tq, const Dims& d,
                      const uint16_t* q,
                      const int32_t* ctx, float* scores, int row0, int rows, int* ticket, int* sched, int32_t* sel,
                      float* sel_score, int32_t* st, int32_t* lu, int32_t step, const int32_t* step_dev, int32_t* fs,
                      int32_t* fb, int32_t* nf, cudaStream_t s) {
    if (rows <= 16)
        return launch_fused<16, kScored>(tmax, tmin, tq, d, q, ctx, scores, row0, rows, ticket, sched, sel, sel_score, st, lu,
                                         step, step_dev, fs, fb, nf, s);
    if (rows <= 32)
        return launch_fused<32, kScored>(tmax, tmin, tq, d, q, ctx, scores, row0, rows, ticket, sched, sel, sel_score, st, lu,
                                         step, step_dev, fs, fb, nf, s);
    if (rows <= 48)
        return launch_fused<48, kScored>(tmax, tmin, tq, d, q, ctx, scores, row0, rows, ticket, sched, sel, sel_score, st, lu,
                                         step, step_dev, fs, fb, nf, s);
    return launch_fused<64, kScored>(tmax, tmin, tq, d, q, ctx, scores, row0, rows, ticket, sched, sel, sel_score, st, lu, step,
                                     step_dev, fs, fb, nf, s);
}

}  // namespace

// Built-in scratch for oasis_score_select_noalloc: the fp32 block scores of
// one call, at most kNoAllocScoreFloats of them.  Every device that loads the
// library holds this array until the process exits.
constexpr size_t kNoAllocScoreFloats = size_t(1) << 20;   // 4 MiB
static __device__ __align__(256) float g_noalloc_scores[kNoAllocScoreFloats];

namespace {

// Device address of g_noalloc_scores on the current device.  In host code the
// array's name is only a stand-in, so the address is looked up once per
// device (with that device current) and cached.
int noalloc_scores(float** out) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static float* cached[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(OASIS_EINVAL, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scores);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(noalloc scratch)");
        cached[dev] = static_cast<float*>(p);
    }
    *out = cached[dev];
    return OASIS_OK;
}

// Scores with query rows [row_begin, row_begin + row_count) of each sequence.
int scores_rows(const oasis_dims* dp, const void* q, int row_begin, int row_count, const void* kmin, const void* kmax,
                const int32_t* ctx_len, float* scores, void* stream) {
    Dims d;
    if (int rc = validate(dp, &d)) return rc;
    if (int rc = check_ptr(q, "q")) return rc;
    if (int rc = check_ptr(kmin, "kmin")) return rc;
    if (int rc = check_ptr(kmax, "kmax")) return rc;
    if (int rc = check_ptr(ctx_len, "ctx_len")) return rc;
    if (int rc = check_ptr(scores, "scores")) return rc;
    if (row_begin < 0 || row_count < 1 || row_begin + row_count > d.Qn)
        return fail(OASIS_EINVAL, "query rows [%d, %d) outside [0, %d)", row_begin, row_begin + row_count, d.Qn);
    const int rows = row_count * d.G();
    const unsigned long long total_rows = static_cast<unsigned long long>(d.B) * d.Hkv * d.N;
    CUtensorMap tmax, tmin;
    if (int rc = make_map(&tmax, kmax, total_rows, oasis::kScoreTile, "kmax")) return rc;
    if (int rc = make_map(&tmin, kmin, total_rows, oasis::kScoreTile, "kmin")) return rc;
    const auto* qq = static_cast<const uint16_t*>(q);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (rows <= 16) return launch_score<16>(tmax, tmin, d, qq, ctx_len, scores, row_begin, rows, s);
    if (rows <= 32) return launch_score<32>(tmax, tmin, d, qq, ctx_len, scores, row_begin, rows, s);
    if (rows <= 48) return launch_score<48>(tmax, tmin, d, qq, ctx_len, scores, row_begin, rows, s);
    return launch_score<64>(tmax, tmin, d, qq, ctx_len, scores, row_begin, rows, s);
}

// Residency diff + capped fetch plan; LRU victims, or by score if scores != NULL;
// the step from step_dev (device) if that is not NULL.
int plan(const oasis_dims* dp, const int32_t* sel, const float* scores, int32_t* slot_table, int32_t* last_used,
         int32_t step, const int32_t* step_dev, int32_t* fetch_slot, int32_t* fetch_block, int32_t* n_fetch,
         void* stream) {
    Dims d;
    if (int rc = validate(dp, &d)) return rc;
    if (int rc = check_ptr(sel, "sel")) return rc;
    if (int rc = check_ptr(slot_table, "slot_table")) return rc;
    if (int rc = check_ptr(last_used, "last_used")) return rc;
    if (int rc = check_ptr(n_fetch, "n_fetch")) return rc;
    if (d.C > 0) {
        if (int rc = check_ptr(fetch_slot, "fetch_slot")) return rc;
        if (int rc = check_ptr(fetch_block, "fetch_block")) return rc;
    }
    const int smem = oasis::plan_smem_ints(d.K) * static_cast<int>(sizeof(int32_t));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (scores != nullptr) {
        if (int rc = set_smem(oasis::plan_fetch_kernel<true>, smem, "plan smem")) return rc;
        oasis::plan_fetch_kernel<true><<<d.B * d.Hkv, oasis::kPlanThreads, smem, s>>>(
            d, sel, scores, slot_table, last_used, step, step_dev, fetch_slot, fetch_block, n_fetch);
    } else {
        if (int rc = set_smem(oasis::plan_fetch_kernel<false>, smem, "plan smem")) return rc;
        oasis::plan_fetch_kernel<false><<<d.B * d.Hkv, oasis::kPlanThreads, smem, s>>>(
            d, sel, scores, slot_table, last_used, step, step_dev, fetch_slot, fetch_block, n_fetch);
    }
    return check_launch("plan_fetch launch");
}

}  // namespace

extern "C" {

const char* oasis_last_error(void) { return g_msg; }

const char* oasis_version(void) { return "oasis-b200 0.1 (sm_100a)"; }

int oasis_check_dims(const oasis_dims* d) { return validate(d, nullptr); }

size_t oasis_workspace_bytes(const oasis_dims* dp) {
    Dims d;
    if (validate(dp, &d) != OASIS_OK) return 0;
    return ws_layout(d).total;
}

int oasis_build_summaries(const oasis_dims* dp, const void* kv, const int32_t* ctx_len, int32_t first_block,
                          int32_t n_blocks, void* kmin, void* kmax, void* stream) {
    Dims d;
    if (int rc = validate(dp, &d)) return rc;
    if (int rc = check_ptr(kv, "kv")) return rc;
    if (int rc = check_ptr(ctx_len, "ctx_len", false)) return rc;
    if (int rc = check_ptr(kmin, "kmin")) return rc;
    if (int rc = check_ptr(kmax, "kmax")) return rc;
    if (first_block < 0 || n_blocks < 0 || first_block + static_cast<long long>(n_blocks) > d.N)
        return fail(OASIS_EINVAL, "block range [%d, %d) outside [0, %d)", first_block, first_block + n_blocks, d.N);
    if (n_blocks == 0) return OASIS_OK;
    const void* src = nullptr;
    if (int rc = device_view(kv, "kv", true, &src)) return rc;
    const long long items = static_cast<long long>(d.B) * d.Hkv * n_blocks;
    const long long grid = (items + oasis::kSumGroups - 1) / oasis::kSumGroups;
    if (grid > 0x7FFFFFFFll) return fail(OASIS_EINVAL, "too many blocks");
    if (int rc = carveout(oasis::build_summaries_kernel, "summaries carve-out")) return rc;
    oasis::build_summaries_kernel<<<static_cast<unsigned>(grid), oasis::kSumThreads, 0,
                                    static_cast<cudaStream_t>(stream)>>>(
        d, static_cast<const uint4*>(src), ctx_len, first_block, n_blocks, static_cast<uint4*>(kmin),
        static_cast<uint4*>(kmax));
    return check_launch("build_summaries launch");
}

int oasis_append_kv(const oasis_dims* dp, const void* k_new, const void* v_new, const int32_t* ctx_len,
                    int32_t* ctx_len_out, void* host_kv, void* kmin, void* kmax, const int32_t* slot_table,
                    void* pool, void* stream) {
    Dims d;
    if (int rc = validate(dp, &d)) return rc;
    if (int rc = check_ptr(k_new, "k_new")) return rc;
    if (int rc = check_ptr(v_new, "v_new")) return rc;
    if (int rc = check_ptr(ctx_len, "ctx_len")) return rc;
    if (int rc = check_ptr(ctx_len_out, "ctx_len_out", true)) return rc;
    if (int rc = check_ptr(host_kv, "host_kv", true)) return rc;
    if (int rc = check_ptr(kmin, "kmin")) return rc;
    if (int rc = check_ptr(kmax, "kmax")) return rc;
    if (int rc = check_ptr(pool, "pool", true)) return rc;
    if (pool != nullptr)
        if (int rc = check_ptr(slot_table, "slot_table")) return rc;
    if (ctx_len_out != nullptr && ctx_len_out == ctx_len)
        return fail(OASIS_EINVAL, "ctx_len_out must not alias ctx_len");
    const void* hv = nullptr;
    if (host_kv != nullptr)
        if (int rc = device_view(host_kv, "host_kv", false, &hv)) return rc;
    if (int rc = carveout(oasis::append_kv_kernel, "append carve-out")) return rc;
    oasis::append_kv_kernel<<<d.B * d.Hkv, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        d, static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), ctx_len, ctx_len_out,
        static_cast<uint4*>(const_cast<void*>(hv)), static_cast<uint4*>(kmin), static_cast<uint4*>(kmax), slot_table,
        static_cast<uint4*>(pool));
    return check_launch("append_kv launch");
}

int oasis_lookahead_scores(const oasis_dims* dp, const void* q, const void* kmin, const void* kmax,
                           const int32_t* ctx_len, float* scores, void* stream) {
    if (dp == nullptr) return fail(OASIS_EINVAL, "dims is NULL");
    const int qn = dp->n_queries;
    return scores_rows(dp, q, qn > 1 ? 1 : 0, qn > 1 ? qn - 1 : 1, kmin, kmax, ctx_len, scores, stream);
}

int oasis_select_topk(const oasis_dims* dp, const float* scores, const int32_t* ctx_len, int32_t* sel,
                      float* sel_score, void* stream) {
    Dims d;
    if (int rc = validate(dp, &d)) return rc;
    if (int rc = check_ptr(scores, "scores")) return rc;
    if (int rc = check_ptr(ctx_len, "ctx_len")) return rc;
    if (int rc = check_ptr(sel, "sel")) return rc;
    if (int rc = check_ptr(sel_score, "sel_score", true)) return rc;
    oasis::select_topk_kernel<<<d.B * d.Hkv, oasis::kSelThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        d, scores, ctx_len, sel, sel_score);
    return check_launch("select_topk launch");
}

int oasis_score_select(const oasis_dims* dp, const void* q, const void* kmin, const void* kmax,
                       const int32_t* ctx_len, int32_t* sel, float* sel_score, void* ws, size_t ws_bytes,
                       void* stream) {
    Dims d;
    if (int rc = validate(dp, &d)) return rc;
    if (int rc = check_ptr(ws, "ws")) return rc;
    const WsLayout w = ws_layout(d);
    if (ws_bytes < w.total) return fail(OASIS_EINVAL, "workspace too small: %zu < %zu", ws_bytes, w.total);
    float* scores = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + w.scores);
    if (int rc = oasis_lookahead_scores(dp, q, kmin, kmax, ctx_len, scores, stream)) return rc;
    return oasis_select_topk(dp, scores, ctx_len, sel, sel_score, stream);
}

int oasis_score_select_rows(const oasis_dims* dp, const void* q, int32_t row_begin, int32_t row_count,
                            const void* kmin, const void* kmax, const int32_t* ctx_len, int32_t* sel,
                            float* sel_score, void* ws, size_t ws_bytes, void* stream) {
    Dims d;
    if (int rc = validate(dp, &d)) return rc;
    if (int rc = check_ptr(ws, "ws")) return rc;
    const WsLayout w = ws_layout(d);
    if (ws_bytes < w.total) return fail(OASIS_EINVAL, "workspace too small: %zu < %zu", ws_bytes, w.total);
    float* scores = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + w.scores);
    if (int rc = scores_rows(dp, q, row_begin, row_count, kmin, kmax, ctx_len, scores, stream)) return rc;
    return oasis_select_topk(dp, scores, ctx_len, sel, sel_score, stream);
}

int oasis_score_select_plan(const oasis_dims* dp, const void* q, const void* kmin, const void* kmax,
                            const int32_t* ctx_len, int32_t* sel, float* sel_score, float* scores,
                            int32_t* slot_table, int32_t* last_used, int32_t step, const int32_t* step_dev,
                            int32_t* fetch_slot, int32_t* fetch_block, int32_t* n_fetch, void* ws, size_t ws_bytes,
                            void* stream) {
    Dims d;
    if (int rc = validate(dp, &d)) return rc;
    if (int rc = check_ptr(q, "q")) return rc;
    if (int rc = check_ptr(kmin, "kmin")) return rc;
    if (int rc = check_ptr(kmax, "kmax")) return rc;
    if (int rc = check_ptr(ctx_len, "ctx_len")) return rc;
    if (int rc = check_ptr(sel, "sel")) return rc;
    if (int rc = check_ptr(sel_score, "sel_score", true)) return rc;
    if (int rc = check_ptr(scores, "scores", true)) return rc;
    if (int rc = check_ptr(slot_table, "slot_table")) return rc;
    if (int rc = check_ptr(last_used, "last_used")) return rc;
    if (int rc = check_ptr(step_dev, "step_dev", true)) return rc;
    if (int rc = check_ptr(n_fetch, "n_fetch")) return rc;
    if (d.C > 0) {
        if (int rc = check_ptr(fetch_slot, "fetch_slot")) return rc;
        if (int rc = check_ptr(fetch_block, "fetch_block")) return rc;
    }
    if (int rc = check_ptr(ws, "ws")) return rc;
    const WsLayout w = ws_layout(d);
    if (ws_bytes < w.total) return fail(OASIS_EINVAL, "workspace too small: %zu < %zu", ws_bytes, w.total);
    uint8_t* base = static_cast<uint8_t*>(ws);
    float* sc = scores != nullptr ? scores : reinterpret_cast<float*>(base + w.scores);
    int* ticket = reinterpret_cast<int*>(base + w.sticket);
    int* sched = reinterpret_cast<int*>(base + w.ssched);
    const int row0 = d.Qn > 1 ? 1 : 0;
    const int rows = (d.Qn > 1 ? d.Qn - 1 : 1) * d.G();
    const unsigned long long total_rows = static_cast<unsigned long long>(d.B) * d.Hkv * d.N;
    CUtensorMap tmax, tmin;
    if (int rc = make_map(&tmax, kmax, total_rows, oasis::kScoreTile, "kmax")) return rc;
    if (int rc = make_map(&tmin, kmin, total_rows, oasis::kScoreTile, "kmin")) return rc;
    CUtensorMap tq;
    if (int rc = make_map_q(&tq, q, d, rows / d.G())) return rc;
    const auto* qq = static_cast<const uint16_t*>(q);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (scores != nullptr)
        return launch_fused_rows<true>(tmax, tmin, tq, d, qq, ctx_len, sc, row0, rows, ticket, sched, sel, sel_score,
                                       slot_table, last_used, step, step_dev, fetch_slot, fetch_block, n_fetch, s);
    return launch_fused_rows<false>(tmax, tmin, tq, d, qq, ctx_len, sc, row0, rows, ticket, sched, sel, sel_score, slot_table,
                                    last_used, step, step_dev, fetch_slot, fetch_block, n_fetch, s);
}

int oasis_block_overlap(const oasis_dims* dp, const int32_t* a, const int32_t* b, int32_t* count, void* stream) {
    Dims d;
    if (int rc = validate(dp, &d)) return rc;
    if (int rc = check_ptr(a, "a")) return rc;
    if (int rc = check_ptr(b, "b")) return rc;
    if (int rc = check_ptr(count, "count")) return rc;
    const int smem = 2 * ((d.N + 31) / 32) * static_cast<int>(sizeof(uint32_t));
    if (int rc = carveout(oasis::block_overlap_kernel, "overlap carve-out")) return rc;
    oasis::block_overlap_kernel<<<d.B * d.Hkv, oasis::kOverlapThreads, smem, static_cast<cudaStream_t>(stream)>>>(
        d, a, b, count);
    return check_launch("block_overlap launch");
}

int oasis_plan_fetch(const oasis_dims* dp, const int32_t* sel, int32_t* slot_table, int32_t* last_used,
                     int32_t step, int32_t* fetch_slot, int32_t* fetch_block, int32_t* n_fetch, void* stream) {
    return plan(dp, sel, nullptr, slot_table, last_used, step, nullptr, fetch_slot, fetch_block, n_fetch, stream);
}

int oasis_plan_fetch_scored(const oasis_dims* dp, const int32_t* sel, const float* scores, int32_t* slot_table,
                            int32_t* last_used, int32_t step, int32_t* fetch_slot, int32_t* fetch_block,
                            int32_t* n_fetch, void* stream) {
    if (int rc = check_ptr(scores, "scores")) return rc;
    return plan(dp, sel, scores, slot_table, last_used, step, nullptr, fetch_slot, fetch_block, n_fetch, stream);
}

int oasis_plan_fetch_at(const oasis_dims* dp, const int32_t* sel, const float* scores, int32_t* slot_table,
                        int32_t* last_used, const int32_t* step, int32_t* fetch_slot, int32_t* fetch_block,
                        int32_t* n_fetch, void* stream) {
    if (int rc = check_ptr(step, "step")) return rc;
    if (int rc = check_ptr(scores, "scores", true)) return rc;
    return plan(dp, sel, scores, slot_table, last_used, 0, step, fetch_slot, fetch_block, n_fetch, stream);
}

int oasis_evict_slots(const oasis_dims* dp, const uint8_t* mask, int32_t* slot_table, void* stream) {
    Dims d;
    if (int rc = validate(dp, &d)) return rc;
    if (int rc = check_ptr(mask, "mask")) return rc;
    if (int rc = check_ptr(slot_table, "slot_table")) return rc;
    const long long n = static_cast<long long>(d.B) * d.Hkv * d.K;
    const unsigned grid = static_cast<unsigned>(std::min<long long>((n + 255) / 256, 4 * 148));
    if (int rc = carveout(oasis::evict_slots_kernel, "evict carve-out")) return rc;
    oasis::evict_slots_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(n, mask, slot_table);
    return check_launch("evict_slots launch");
}

namespace {

int ev_record(void* ev, void* stream, const char* what) {
    if (ev == nullptr) return OASIS_OK;
    const cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(ev), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? OASIS_OK : cuda_fail(e, what);
}

int ev_wait(void* stream, void* ev, const char* what) {
    const cudaError_t e = cudaStreamWaitEvent(static_cast<cudaStream_t>(stream), static_cast<cudaEvent_t>(ev), 0);
    return e == cudaSuccess ? OASIS_OK : cuda_fail(e, what);
}

}  // namespace

int oasis_decode_layer_step(const oasis_dims* dp, const oasis_layer* L, const void* q, const int32_t* ctx_len,
                            const uint8_t* evict_mask, int32_t step, const int32_t* step_dev, float scale, void* ws,
                            size_t ws_bytes, const oasis_step_sync* S) {
    if (L == nullptr || S == nullptr) return fail(OASIS_EINVAL, "layer and sync must not be NULL");
    if (S->fetch_done == nullptr || S->plan_ready == nullptr)
        return fail(OASIS_EINVAL, "fetch_done and plan_ready events must be given");
    int rc;
    if (!S->in_graph && (rc = ev_wait(S->main, S->fetch_done, "wait fetch_done"))) return rc;
    // attention over the working set staged by the previous step
    if ((rc = ev_record(S->timing[0], S->main, "timing"))) return rc;
    if ((rc = oasis_sparse_attn(dp, q, L->pool, L->slot_table, ctx_len, scale, L->out, L->lse, ws, ws_bytes,
                                S->main)))
        return rc;
    if ((rc = ev_record(S->timing[1], S->main, "timing"))) return rc;
    if (evict_mask != nullptr && (rc = oasis_evict_slots(dp, evict_mask, L->slot_table, S->main))) return rc;
    // lookahead scores + top-K + residency diff and capped plan, one launch,
    // after the attention that read this layer's slot table
    if ((rc = ev_record(S->timing[2], S->main, "timing"))) return rc;
    if ((rc = oasis_score_select_plan(dp, q, L->kmin, L->kmax, ctx_len, L->sel, L->sel_score, L->scores,
                                      L->slot_table, L->last_used, step, step_dev, L->fetch_slot, L->fetch_block,
                                      L->n_fetch, ws, ws_bytes, S->main)))
        return rc;
    if ((rc = ev_record(S->timing[3], S->main, "timing"))) return rc;
    if ((rc = ev_record(S->plan_ready, S->main, "record plan_ready")) ||
        (rc = ev_wait(S->copy, S->plan_ready, "wait plan_ready")))
        return rc;
    // the gather of the missing blocks, on the copy stream
    if ((rc = ev_record(S->timing[4], S->copy, "timing"))) return rc;
    if ((rc = oasis_prefetch(dp, L->host_kv, L->fetch_slot, L->fetch_block, L->n_fetch, L->pool, S->copy))) return rc;
    if ((rc = ev_record(S->timing[5], S->copy, "timing"))) return rc;
    return ev_record(S->fetch_done, S->copy, "record fetch_done");
}

int oasis_step_advance(int32_t* step, void* stream) {
    if (int rc = check_ptr(step, "step")) return rc;
    if (int rc = carveout(oasis::step_advance_kernel, "step carve-out")) return rc;
    oasis::step_advance_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(step);
    return check_launch("step_advance launch");
}

int oasis_prefetch(const oasis_dims* dp, const void* host_kv, const int32_t* fetch_slot, const int32_t* fetch_block,
                   const int32_t* n_fetch, void* pool, void* stream) {
    Dims d;
    if (int rc = validate(dp, &d)) return rc;
    if (int rc = check_ptr(host_kv, "host_kv")) return rc;
    if (int rc = check_ptr(n_fetch, "n_fetch")) return rc;
    if (int rc = check_ptr(pool, "pool")) return rc;
    if (d.C == 0) return OASIS_OK;
    if (int rc = check_ptr(fetch_slot, "fetch_slot")) return rc;
    if (int rc = check_ptr(fetch_block, "fetch_block")) return rc;
    const void* hv = nullptr;
    if (int rc = device_view(host_kv, "host_kv", false, &hv)) return rc;
    const long long entries = static_cast<long long>(d.B) * d.Hkv * d.C;
    const unsigned grid = static_cast<unsigned>(std::min<long long>(oasis::kPrefetchCtas, (entries + 1) / 2));
    if (int rc = carveout(oasis::prefetch_kernel, "prefetch carve-out")) return rc;
    oasis::prefetch_kernel<<<grid, oasis::kPrefetchThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        d, static_cast<const uint4*>(hv), fetch_slot, fetch_block, n_fetch, static_cast<uint4*>(pool));
    return check_launch("prefetch launch");
}

int oasis_sparse_attn(const oasis_dims* dp, const void* q, const void* pool, const int32_t* slot_table,
                      const int32_t* ctx_len, float scale, float* out, float* lse, void* ws, size_t ws_bytes,
                      void* stream) {
    Dims d;
    if (int rc = validate(dp, &d)) return rc;
    if (int rc = check_ptr(q, "q")) return rc;
    if (int rc = check_ptr(pool, "pool")) return rc;
    if (int rc = check_ptr(slot_table, "slot_table")) return rc;
    if (int rc = check_ptr(ctx_len, "ctx_len")) return rc;
    if (int rc = check_ptr(out, "out")) return rc;
    if (int rc = check_ptr(lse, "lse")) return rc;
    if (int rc = check_ptr(ws, "ws")) return rc;
    if (!(scale > 0.f) || !(scale < 3.0e38f)) return fail(OASIS_EINVAL, "scale must be a positive finite float");
    const WsLayout w = ws_layout(d);
    if (ws_bytes < w.total) return fail(OASIS_EINVAL, "workspace too small: %zu < %zu", ws_bytes, w.total);
    CUtensorMap tk, tv, tq;
    const unsigned long long slots = static_cast<unsigned long long>(d.B) * d.Hkv * d.K;
    if (int rc = make_map_pool(&tk, pool, slots, "pool keys")) return rc;
    if (int rc = make_map_pool(&tv, static_cast<const uint8_t*>(pool) + oasis::kBlockBytes / 2, slots, "pool values"))
        return rc;
    if (int rc = make_map_q(&tq, q, d, d.Qn)) return rc;
    uint8_t* base = static_cast<uint8_t*>(ws);
    float* ws_lse = reinterpret_cast<float*>(base + w.lse);
    float* ws_o = reinterpret_cast<float*>(base + w.o);
    int* ws_ticket = reinterpret_cast<int*>(base + w.ticket);
    int* ws_sched = reinterpret_cast<int*>(base + w.sched);
    const float scale_log2 = scale * 1.4426950408889634f;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const oasis::AttnChunks chunks = attn_chunks(d, sm_count());
    // An attention CTA fills an SM's register file, so no gather CTA fits
    // beside it: leave the gather's SMs free, so a gather on the copy stream
    // keeps running while the attention of another layer does (the chunks
    // are taken from a counter, so fewer CTAs only take more chunks each).
    const int grid_max = std::max(1, sm_count() - oasis::kPrefetchCtas);
    const unsigned ctas = static_cast<unsigned>(std::min(grid_max, chunks.nc));
    const bool r32 = d.Qn * d.G() <= 32;
    auto kern = r32 ? oasis::sparse_attn_kernel<32> : oasis::sparse_attn_kernel<64>;
    const int smem = oasis::attn_smem(r32 ? 32 : 64);
    if (int rc = set_smem(kern, smem, "sparse_attn smem")) return rc;
    kern<<<ctas, oasis::kAttnThreads, smem, s>>>(tk, tv, tq, d, slot_table, ctx_len, scale_log2, chunks,
                                                             out, lse, ws_o, ws_lse, ws_ticket, ws_sched);
    return check_launch("sparse_attn launch");
}

int oasis_read_device_error(uint32_t* out, int clear, void* stream) {
    if (out == nullptr) return fail(OASIS_EINVAL, "out is NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, oasis::g_oasis_dev_error, sizeof(v), 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "read device error");
    if (clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbolAsync(oasis::g_oasis_dev_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return cuda_fail(e, "clear device error");
    }
    *out = v;
    return OASIS_OK;
}

int oasis_score_select_noalloc(const oasis_dims* dp, const void* q, const void* kmin, const void* kmax,
                               const int32_t* ctx_len, int32_t* sel, float* sel_score, void* stream) {
    Dims d;
    if (int rc = validate(dp, &d)) return rc;
    const size_t n = static_cast<size_t>(d.B) * d.Hkv * d.N;
    if (n > kNoAllocScoreFloats)
        return fail(OASIS_EINVAL,
                    "batch * n_kv_heads * max_blocks = %zu exceeds the built-in scratch of %zu block scores (4 MiB); "
                    "use oasis_score_select with a workspace",
                    n, kNoAllocScoreFloats);
    float* scores = nullptr;
    if (int rc = noalloc_scores(&scores)) return rc;
    // No entry needs to start at zero: the scorer writes every valid block's
    // score before the selector reads it, and nothing else is read.
    if (int rc = oasis_lookahead_scores(dp, q, kmin, kmax, ctx_len, scores, stream)) return rc;
    return oasis_select_topk(dp, scores, ctx_len, sel, sel_score, stream);
}

}  // extern "C"
