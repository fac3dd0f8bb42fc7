/*
 * oasis.h - C ABI of the B200 lookahead sparse-KV decode path (liboasis.so).
 *
 * The library implements the decode-time hot path described on the page
 * "OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
 * Prefetching" (metalmedia.ai explainer of arXiv 2608.08097): draft queries
 * from speculative decoding score every paged KV block against per-block key
 * min/max summaries (Figure 7), the top blocks under a token budget are
 * selected (Figure 7; "What they did", item 4), only the selected blocks that
 * are not resident in the HBM pool are copied in from pinned host memory,
 * capped per step (method sketch item 3; Table 2; "Terms in this paper":
 * capped eviction), through a per-KV-head slot table (Figure 9), and GQA
 * attention runs for the 1+k verification/draft queries over the resident
 * blocks only (Figure 7, right).  The pipeline order across steps follows
 * Figure 8.  The block scorer is Quest's per-channel upper bound (the page
 * "Quest: Query-Aware Sparsity for Efficient Long-Context LLM Inference",
 * cited among the paper's references), because the OasisKV pages name the
 * min/max pooling but print no scoring formula.
 *
 * Conventions for every entry point
 *   - All pointers are caller-owned.  The library allocates no memory on any
 *     call listed here; it keeps one 32-bit device error word per device.
 *   - "device" pointers must be CUDA device memory of the current device;
 *     "mapped host" pointers must be pinned host memory that the current
 *     device can address (cudaHostAlloc / cudaHostRegister, or a pinned
 *     torch tensor on a UVA system).  Every pointer must be 16-byte aligned.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous: no entry point synchronises except
 *     oasis_read_device_error.
 *   - Return value: OASIS_OK, or a negative code; the message of the last
 *     failure on the calling thread is oasis_last_error().  Argument errors
 *     are detected on the host before anything is enqueued.  Out-of-range ids
 *     found on the device (slot table or selection entries, append positions)
 *     are skipped by the kernels and recorded in the device error word;
 *     kernels never trap.
 *
 * Layouts (row-major, innermost last; bf16 = IEEE bfloat16 bit patterns)
 *   q          bf16  [B][Qn][Hq][D]   row j=0 verification query, j>=1 drafts
 *   host KV    bf16  [B][Hkv][N][2][P][D]   per block: P key rows, P value rows
 *   pool       bf16  [B][Hkv][K][2][P][D]   fixed HBM working set, one slot per
 *                                          block; slot s of (b,h) holds block
 *                                          slot_table[b][h][s] (or is free: -1)
 *   kmin,kmax  bf16  [B][Hkv][N][D]   per-block per-channel key min / max
 *   ctx_len    int32 [B]              valid context tokens of each sequence
 *   slot_table int32 [B][Hkv][K]      block id held by each pool slot, or -1
 *   last_used  int32 [B][Hkv][K]      step at which the slot's block was last
 *                                     selected or fetched
 *   sel        int32 [B][Hkv][K]      selected block ids, rank order, -1 padded
 *   fetch_slot, fetch_block  int32 [B][Hkv][C];  n_fetch int32 [B][Hkv]
 *   out        fp32  [B][Qn][Hq][D];  lse fp32 [B][Qn][Hq] (natural log)
 *
 * Fixed sizes: D = 128, P = 16.  Limits: 1 <= Hkv, Hq % Hkv == 0,
 * 1 <= K <= 1024, K <= N <= 32768, 0 <= C <= K, 1 <= Qn,
 * Qn*G <= 64 (attention rows per KV head), max(1,Qn-1)*G <= 64 (scoring rows).
 */
#ifndef OASIS_H
#define OASIS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct oasis_dims {
    int32_t batch;         /* B  */
    int32_t n_q_heads;     /* Hq */
    int32_t n_kv_heads;    /* Hkv; G = Hq / Hkv query heads share one KV head */
    int32_t head_dim;      /* D, must be 128 */
    int32_t block_tokens;  /* P, must be 16 */
    int32_t max_blocks;    /* N: block capacity of each (sequence, KV head) */
    int32_t budget_blocks; /* K: token budget / P = pool slots per (sequence, KV head) */
    int32_t n_queries;     /* Qn = 1 + k (verification + drafts) */
    int32_t fetch_cap;     /* C: most blocks fetched per (sequence, KV head) per step */
} oasis_dims;

enum {
    OASIS_OK = 0,
    OASIS_EINVAL = -1,     /* bad dims, null / misaligned pointer, workspace too small */
    OASIS_ENOTMAPPED = -2, /* a host pointer the device cannot address */
    OASIS_ECUDA = -3,      /* a CUDA runtime / driver call or launch failed */
    OASIS_ERANGE = -4      /* reserved for device-detected range errors (see error word) */
};

/* Bits of the device error word (oasis_read_device_error). */
#define OASIS_DEVERR_ID_RANGE    0x1u  /* slot-table / selection / fetch id out of [0, N) or [0, K) */
#define OASIS_DEVERR_TIMEOUT     0x2u  /* a bounded barrier wait gave up; the kernel returned early */
#define OASIS_DEVERR_APPEND_FULL 0x4u  /* append position at or beyond N * P */
#define OASIS_DEVERR_DUPLICATE   0x8u  /* a block resident twice / selected twice */

/* Workspace bytes needed by oasis_score_select, oasis_score_select_plan and
 * oasis_sparse_attn for these dims (the scoring and the attention use
 * separate regions, so they may run concurrently on different streams with
 * the same workspace; two attention calls, or two scoring calls, on one
 * workspace must be stream-ordered).  The workspace is device memory that
 * must be zero-filled once before its first use; the kernels leave it ready
 * for the next call.  One workspace per concurrently running layer. */
size_t oasis_workspace_bytes(const oasis_dims* d);

/* a1 - block summaries (OasisKV Figure 7, left: compressed keys by per-block
 * min/max pooling).  For blocks n in [first_block, first_block + n_blocks)
 * with at least one valid token (n*P < ctx_len[b]), writes
 *   kmin[b][h][n][c] = min over valid tokens t of K[b][h][n][t][c], kmax = max.
 * Blocks without a valid token are left untouched.  kv: device or mapped
 * host, layout of host KV.  ctx_len, kmin, kmax: device. */
int oasis_build_summaries(const oasis_dims* d, const void* kv, const int32_t* ctx_len,
                          int32_t first_block, int32_t n_blocks,
                          void* kmin, void* kmax, void* stream);

/* a1 (append) - one decoded token per sequence.  For every (b, h) the new
 * key / value rows k_new, v_new (device, bf16 [B][Hkv][D]) go to position
 * p = ctx_len[b] (device): written into host_kv (mapped host; may be NULL to
 * skip), folded into kmin/kmax of block p / P (overwrite when p opens the
 * block, running min/max otherwise), and written into the pool slot that
 * holds block p / P if it is resident (slot_table, pool: device; pool may be
 * NULL).  If ctx_len_out is not NULL, ctx_len_out[b] = ctx_len[b] + 1
 * (it must not alias ctx_len).  Positions >= N*P set OASIS_DEVERR_APPEND_FULL. */
int oasis_append_kv(const oasis_dims* d, const void* k_new, const void* v_new,
                    const int32_t* ctx_len, int32_t* ctx_len_out, void* host_kv,
                    void* kmin, void* kmax, const int32_t* slot_table, void* pool,
                    void* stream);

/* a2 - lookahead scores (OasisKV Figure 7, right: the draft queries scan the
 * compressed keys; method sketch item 2).  For every valid block n of (b, h):
 *   scores[b][h][n] = max over draft rows j in [1, Qn) (row 0 if Qn == 1)
 *                     and g < G of  sum_c max(q_c*kmin_c, q_c*kmax_c),
 * q = q[b][j][h*G+g], accumulated in fp32 from exact bf16 products.
 * Entries for blocks n >= ceil(ctx_len[b]/P) are not written.
 * q, kmin, kmax, ctx_len, scores (fp32 [B][Hkv][N]): device. */
int oasis_lookahead_scores(const oasis_dims* d, const void* q, const void* kmin,
                           const void* kmax, const int32_t* ctx_len, float* scores,
                           void* stream);

/* a3 - top-K selection (OasisKV Figure 7: the K blocks the next step uses).
 * Per (b, h): ranks the valid blocks by (score descending, block id
 * ascending; -0.0 == +0.0) and writes the first min(K, n_valid) ids to sel in
 * rank order, -1 padded; sel_score (nullable) gets their scores, -inf padded.
 * scores: device fp32 [B][Hkv][N]; sel, sel_score: device. */
int oasis_select_topk(const oasis_dims* d, const float* scores, const int32_t* ctx_len,
                      int32_t* sel, float* sel_score, void* stream);

/* a2 + a3 - scores into the workspace, then top-K.  ws: device workspace of
 * oasis_workspace_bytes(d) bytes. */
int oasis_score_select(const oasis_dims* d, const void* q, const void* kmin,
                       const void* kmax, const int32_t* ctx_len, int32_t* sel,
                       float* sel_score, void* ws, size_t ws_bytes, void* stream);

/* a2 + a3 over a chosen range of query rows: the scores take the max over
 * rows j in [row_begin, row_begin + row_count) (and the G heads) instead of
 * the drafts, then top-K as oasis_select_topk.  row_begin = 0, row_count = 1
 * ranks the blocks for the verification query alone: the exact top-K set of
 * the true query (OasisKV Figure 6) and the previous-token prediction of
 * Figure 4; a corrective fetch plans from it.  Same buffers and workspace as
 * oasis_score_select; EINVAL if the rows fall outside [0, Qn). */
int oasis_score_select_rows(const oasis_dims* d, const void* q, int32_t row_begin,
                            int32_t row_count, const void* kmin, const void* kmax,
                            const int32_t* ctx_len, int32_t* sel, float* sel_score,
                            void* ws, size_t ws_bytes, void* stream);

/* a2 + a3 + a4 in one launch (OasisKV Figure 8: per layer the drafts'
 * prediction, the selection and the residency diff with the capped plan run
 * back to back before the transfer can start).  Results are those of
 * oasis_lookahead_scores, oasis_select_topk and oasis_plan_fetch (scores ==
 * NULL) or oasis_plan_fetch_scored (scores != NULL) called in turn, bit for
 * bit.  scores: NULL keeps the block scores in the workspace; else device fp32
 * [B][Hkv][N] that receives them and orders the victims by score.  step_dev:
 * NULL uses `step`, else the step number is read from device memory at run
 * time (graph capture).  sel_score may be NULL.  Every buffer is device
 * memory; ws: a workspace of oasis_workspace_bytes(d) bytes.  The plan reads
 * and rewrites slot_table / last_used, so it must run after any attention
 * that reads this layer's slot table.  EINVAL also when the fused kernel's
 * shared memory cannot hold one unit's N keys and plan (up to 4*N + 64*K
 * bytes above 226 KiB, i.e. only near N = 32768 with a large K). */
int oasis_score_select_plan(const oasis_dims* d, const void* q, const void* kmin,
                            const void* kmax, const int32_t* ctx_len, int32_t* sel,
                            float* sel_score, float* scores, int32_t* slot_table,
                            int32_t* last_used, int32_t step, const int32_t* step_dev,
                            int32_t* fetch_slot, int32_t* fetch_block, int32_t* n_fetch,
                            void* ws, size_t ws_bytes, void* stream);

/* Prediction quality (OasisKV Figure 4: top-K accuracy of the previous token
 * vs a lookahead token; Figure 6: agreement of the predicted top-K with the
 * exact set).  count[b][h] = number of distinct block ids in b[b][h][0..K)
 * that also occur in a[b][h][0..K); -1 entries are empty.  a, b: device
 * int32 [B][Hkv][K] (selections, exact sets or slot tables); count: device
 * int32 [B][Hkv].  Ids outside [-1, N) are skipped and set
 * OASIS_DEVERR_ID_RANGE. */
int oasis_block_overlap(const oasis_dims* d, const int32_t* a, const int32_t* b,
                        int32_t* count, void* stream);

/* Allocation-free variant of oasis_score_select (no counterpart in the
 * paper; it exists for callers that cannot provide device scratch memory).
 * Some callers cannot allocate or pass a workspace: an attention backend
 * behind an engine interface that hands over only input and output tensors,
 * or a process that reserved its device memory up front, where a cudaMalloc
 * would fail or stall the device in the middle of a decode step.  This entry
 * point takes the same inputs and outputs as oasis_score_select and keeps the
 * block scores in a fixed 4 MiB array compiled into the library instead:
 *   - limit: batch * n_kv_heads * max_blocks <= 1048576 (4 MiB of fp32
 *     scores); larger dims return OASIS_EINVAL with a message;
 *   - it calls no cudaMalloc / cudaFree and no allocating library routine;
 *   - the first call on each device looks up the array's device address
 *     (with that device current) and caches it; make that first call before
 *     any stream capture;
 *   - every call on a device shares the one array, which keeps the last
 *     call's scores; calls whose work overlaps on the GPU (for example on two
 *     streams) race on it and must be serialised by the caller;
 *   - each GPU that loads the library holds the 4 MiB until the process
 *     exits;
 *   - errors: the dims and the scratch limit are checked first, then the
 *     array's address is looked up (OASIS_ECUDA when no device is usable),
 *     then the buffers, as in oasis_lookahead_scores / oasis_select_topk. */
int oasis_score_select_noalloc(const oasis_dims* d, const void* q, const void* kmin,
                               const void* kmax, const int32_t* ctx_len, int32_t* sel,
                               float* sel_score, void* stream);

/* a4 - residency diff and capped fetch plan (OasisKV method sketch item 3;
 * Table 2: LRU eviction; Figure 9: per-head slot table).  Per (b, h), with
 * S* the blocks of sel: slots holding a block of S* get last_used = step;
 * M = blocks of S* not resident, in rank order; the first min(C, |M|) are
 * fetched into victims taken first from free slots (ascending slot), then
 * from slots whose block is not in S*, ordered by (last_used, block id)
 * ascending; each victim gets the new block and last_used = step.
 * Writes fetch_slot / fetch_block (-1 padded) and n_fetch, and updates
 * slot_table / last_used in place.  All pointers device.  Bit-exact. */
int oasis_plan_fetch(const oasis_dims* d, const int32_t* sel, int32_t* slot_table,
                     int32_t* last_used, int32_t step, int32_t* fetch_slot,
                     int32_t* fetch_block, int32_t* n_fetch, void* stream);

/* a4 with score-ordered victims (the eviction ablation's alternative to the
 * LRU order of OasisKV Table 2): as oasis_plan_fetch, except that stale slots
 * are taken by (score of their block, block id) ascending, the lowest-scored
 * block first (-0.0 == +0.0).  scores: device fp32 [B][Hkv][N], this step's
 * lookahead scores (oasis_lookahead_scores); entries of resident blocks must
 * be written (a resident block is always below n_valid). */
int oasis_plan_fetch_scored(const oasis_dims* d, const int32_t* sel, const float* scores,
                            int32_t* slot_table, int32_t* last_used, int32_t step,
                            int32_t* fetch_slot, int32_t* fetch_block, int32_t* n_fetch,
                            void* stream);

/* a4 with the step number in device memory (a7 graph capture: the planner is
 * the only call of a decode step that takes a per-step scalar, so a captured
 * multi-layer step reads it from here and replays unchanged).  As
 * oasis_plan_fetch (scores == NULL) or oasis_plan_fetch_scored (scores
 * given), with step = *step read on the device when the kernel runs.
 * step: device int32, 16-byte aligned. */
int oasis_plan_fetch_at(const oasis_dims* d, const int32_t* sel, const float* scores,
                        int32_t* slot_table, int32_t* last_used, const int32_t* step,
                        int32_t* fetch_slot, int32_t* fetch_block, int32_t* n_fetch,
                        void* stream);

/* Residency loss (the 32K Qwen3-32B configuration: a seeded share of the
 * attended KV misses residency each step; no counterpart in the method
 * itself, it models blocks lost to memory pressure): slot_table[i] = -1
 * wherever mask[i] != 0.  mask: device uint8 [B][Hkv][K]; slot_table:
 * device int32 [B][Hkv][K], updated in place.  Call it after a layer's
 * attention and before its plan, so a lost block that is selected again is
 * fetched again. */
int oasis_evict_slots(const oasis_dims* d, const uint8_t* mask, int32_t* slot_table, void* stream);

/* *step += 1 on the device (one thread), stream-ordered: the first call of a
 * captured decode step. */
int oasis_step_advance(int32_t* step, void* stream);

/* ---- a7: one layer's decode step in a single call ------------------------
 * OasisKV Figure 8: per layer, attention over the resident blocks on the main
 * stream; lookahead scoring and top-K on a second stream concurrent with it;
 * the plan on the main stream once the selection is ready; the gather on a
 * third (high-priority) stream once the plan is ready, landing before that
 * layer's attention at the next step.  This entry point enqueues all of it
 * with the stream / event order done natively (cudaStreamWaitEvent /
 * cudaEventRecord), so a whole layer-step costs the host one call. */

/* One attention layer's buffers; every pointer is device memory unless noted. */
typedef struct oasis_layer {
    const void* host_kv;    /* pinned, mapped host KV [B][Hkv][N][2][P][D] bf16 */
    const void* kmin;       /* [B][Hkv][N][D] bf16 */
    const void* kmax;
    void* pool;             /* [B][Hkv][K][2][P][D] bf16 */
    int32_t* slot_table;    /* [B][Hkv][K] */
    int32_t* last_used;     /* [B][Hkv][K] */
    int32_t* sel;           /* [B][Hkv][K] */
    float* sel_score;       /* [B][Hkv][K], may be NULL */
    float* scores;          /* NULL: scores in the workspace, LRU victims (oasis_plan_fetch);
                               [B][Hkv][N] of this layer: scores kept here, score-ordered
                               victims (oasis_plan_fetch_scored) */
    int32_t* fetch_slot;    /* [B][Hkv][C] */
    int32_t* fetch_block;   /* [B][Hkv][C] */
    int32_t* n_fetch;       /* [B][Hkv] */
    float* out;             /* [B][Qn][Hq][D] fp32 */
    float* lse;             /* [B][Qn][Hq] fp32 */
} oasis_layer;

/* Streams (cudaStream_t; NULL is the default stream) and this layer's events
 * (cudaEvent_t, created by the caller) of a layer-step.  With in_graph set
 * (inside a capture of a whole step) the main stream does not wait for
 * fetch_done.  timing: optional begin / end events recorded around the
 * attention (main), the fused scores + top-K + plan (main) and the gather
 * (copy), in that order; NULL entries are skipped. */
typedef struct oasis_step_sync {
    void* main;
    void* copy;
    void* fetch_done;       /* recorded on copy after the gather */
    void* plan_ready;       /* recorded on main after the plan */
    int32_t in_graph;
    void* timing[6];
} oasis_step_sync;

/* Decode step `step` of one layer, in the order above: [wait fetch_done] ->
 * attention(q, scale) -> [residency loss: evict_mask, may be NULL] -> scores +
 * top-K + plan in one launch (oasis_score_select_plan; step number `step`, or
 * *step_dev when step_dev != NULL) -> gather on copy.  Same buffers,
 * workspace and results as the individual calls; the first error returns
 * before anything after it is enqueued.  Everything but the gather runs on
 * main, so queries written on main before the call are ordered before both
 * readers. */
int oasis_decode_layer_step(const oasis_dims* d, const oasis_layer* layer, const void* q,
                            const int32_t* ctx_len, const uint8_t* evict_mask, int32_t step,
                            const int32_t* step_dev, float scale, void* ws, size_t ws_bytes,
                            const oasis_step_sync* sync);

/* a5 - host-to-HBM gather (OasisKV Figure 7: the chosen blocks come in from
 * the CPU-side KV cache ahead of use; Figure 8).  For i < n_fetch[b][h], copies the 8 KiB block
 * host_kv[b][h][fetch_block[b][h][i]] into pool[b][h][fetch_slot[b][h][i]]
 * with a kernel that reads the mapped pinned host memory directly over PCIe
 * (no copy-engine call, so it stays stream-ordered after the planner).
 * host_kv: mapped host (OASIS_ENOTMAPPED otherwise); the rest device. */
int oasis_prefetch(const oasis_dims* d, const void* host_kv, const int32_t* fetch_slot,
                   const int32_t* fetch_block, const int32_t* n_fetch, void* pool,
                   void* stream);

/* a6 - sparse GQA decode attention (OasisKV Figure 7, right: the verification
 * query and the drafts attended in one pass over the resident working set).  For every b,
 * row j < Qn and query head hq (KV head h = hq / G): over the valid tokens of
 * every occupied slot of (b, h),
 *   out = sum softmax(scale * q.k) v,   lse = log sum exp(scale * q.k);
 * no occupied slot / no valid token gives out = 0, lse = -inf.  bf16 inputs,
 * fp32 accumulation (the softmax weights enter the P.V product as a bf16
 * head plus a bf16 remainder).  scale must be positive and finite
 * (OASIS_EINVAL otherwise).  q, pool, slot_table, ctx_len, out, lse, ws:
 * device.  Value rows past the context in a partly filled block are never
 * multiplied in (non-finite stale bytes there do not reach out). */
int oasis_sparse_attn(const oasis_dims* d, const void* q, const void* pool,
                      const int32_t* slot_table, const int32_t* ctx_len, float scale,
                      float* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/* Reads (and if clear != 0 resets) this device's error word; synchronises
 * `stream`.  For tests and diagnostics, not for the hot loop. */
int oasis_read_device_error(uint32_t* out, int clear, void* stream);

/* Checks dims against the limits above without touching the device. */
int oasis_check_dims(const oasis_dims* d);

/* Message of the last failure on the calling thread ("" if none). */
const char* oasis_last_error(void);

/* Library version string. */
const char* oasis_version(void);

#ifdef __cplusplus
}
#endif

#endif /* OASIS_H */
