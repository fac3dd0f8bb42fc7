"""Plain CPU oracle for the OasisKV lookahead sparse-KV decode path.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check in
``__graft_entry__``, and the CPU-baseline leg and ``--impl reference`` arm of
``bench.py`` (through ``oracle/decode_timing.py``) may import or run anything
in this package.  The CUDA library never calls into it and shares no
code, header, table or helper with it; the only thing both sides share is the
seeded input generator, which holds none of the method's arithmetic.

Everything here is written for a reader checking it against the pages by eye:
fp64 arithmetic, whole-array numpy where it reads like the formula, plain
Python loops where the step is a procedure (the planner), no blocking, fusion
or reordering beyond what the definitions state.

Sources, cited by page title plus figure / table / section:

* [OasisKV] "OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead
  Sparse Prefetching" (metalmedia.ai explainer of arXiv 2608.08097):
  "What they did" items 2-3, the numbered method sketch (items 2-4),
  Figures 7, 8 and 9, Table 2 and the "Terms in this paper" list.
* [Quest] "Quest: Query-Aware Sparsity for Efficient Long-Context LLM
  Inference" (in the reference list of the mlsanity.com index page of the
  same paper): the per-channel min/max upper bound used as the block scorer.
  The OasisKV pages say the draft query scans keys compressed by per-block
  min/max pooling (Figure 7) but do not print the scoring formula; the
  scorer here is Quest's bound.

Data conventions (all arrays numpy):

* keys / values / queries arrive as float64 arrays holding bf16-exact values
  (``bf16_bits_to_f64`` converts raw bf16 bit patterns).
* ``ctx_len[b]`` is the number of valid context tokens of sequence ``b``;
  block ``n`` of a sequence holds tokens ``n*P .. n*P+P-1``; a token is valid
  when its position is ``< ctx_len[b]``.  ``n_valid(b) = ceil(ctx_len[b]/P)``.
* GQA: query head ``hq`` reads KV head ``hq // G`` with ``G = Hq / Hkv``.
* Query rows ``j = 0 .. Qn-1`` of a decode step: row 0 is the verification
  (normal) query, rows ``1 .. Qn-1`` are the draft queries ([OasisKV] Fig. 7,
  right).  When ``Qn == 1`` there are no drafts and row 0 is used for scoring
  (a degenerate previous-token predictor; see the readings below).

Readings taken where the pages are silent:

* R1 scorer: ``s[n] = max_{j>=1, g<G} sum_c max(q_c*kmin_c, q_c*kmax_c)``,
  no 1/sqrt(D) factor, summed in fp64 and rounded once to fp32.
* R2 ranking: score descending, ties to the lower block index; -0.0 == +0.0.
* R3 fetch order when more than ``C`` blocks are missing: rank order.
* R4 victim order: free slots first (ascending slot), then occupied slots
  whose block is not selected this step, least recently used first, ties to
  the lower block id ([OasisKV] Table 2 names LRU eviction).  A block used
  at step t is one selected at t or fetched at t.
* R5 attention reads every occupied slot (the resident blocks), masking
  tokens at or beyond ``ctx_len``; all ``Qn`` rows see the same token set.
* R6 empty token set: output 0, log-sum-exp -inf.
* R16 exact set and corrective fetch ([OasisKV] Figure 6 and "What they did":
  prediction misses need corrective fetches).  At decode step t the exact
  set E_t is the top-K under the same scorer with the verification row
  (row 0, the true query of step t) alone.  Agreement of a predicted set S
  with E_t is |S & E_t| (reported over |E_t|); the lookahead prediction is
  the selection made from the drafts of step t-1, the previous-token
  prediction is E_{t-1}.  A corrective fetch brings every block of E_t that
  is not resident before step t's attention, with the same planner and no
  cap (C = K), as a use at step t.
* R17 score-based victims (the alternative to Table 2's LRU in the eviction
  ablation): stale slots are taken in order of their block's current
  lookahead score, lowest first, ties to the lower block id (-0.0 == +0.0);
  free slots still come first and a selected block is never evicted.
* R9 appended tokens (the long-output reasoning configuration: one new
  token per sequence per step): the token accepted at step t-1 is written at
  the start of step t, before that layer's attention, at position
  ``ctx_len[b]`` of the host KV, folded into the block summaries, and copied
  into the pool slot that holds its block if that block is resident; the
  context is one token longer from then on.  A token that opens a new block
  is therefore not attended at the step it arrives: its block becomes
  resident only once a plan selects and fetches it (Figure 8 order).
* R19 residency loss (the 32K Qwen3-32B configuration: a seeded share of
  the attended KV misses residency each step): at decode step t, after the
  layer's attention and before its selection / plan, every slot the step's
  mask marks is freed (slot -> -1); a lost block that is selected again is
  a miss and is fetched again.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "bf16_bits_to_f64",
    "f64_to_bf16_bits",
    "n_valid_blocks",
    "block_summaries",
    "summary_append",
    "append_token",
    "lookahead_scores",
    "select_topk",
    "plan_fetch",
    "prefetch",
    "sparse_attention",
    "dense_attention",
    "block_overlap",
    "evict_slots",
    "decode_layer_steps",
]


# ----------------------------------------------------------------- bf16 I/O
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bit patterns (uint16) to float64, exactly."""
    u32 = bits.astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Narrow float64 values that are already bf16-representable to bf16 bits.

    Raises if a value would need rounding: the oracle only ever narrows
    results of min/max over bf16 inputs, which are exact.
    """
    f32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    if not np.array_equal(f32.astype(np.float64), np.asarray(x, np.float64), equal_nan=True):
        raise ValueError("value not representable in fp32")
    u32 = f32.view(np.uint32)
    if np.any((u32 & np.uint32(0xFFFF)) != 0):
        raise ValueError("value not representable in bf16")
    return (u32 >> np.uint32(16)).astype(np.uint16)


def n_valid_blocks(ctx_len: np.ndarray, block_tokens: int) -> np.ndarray:
    """Blocks that hold at least one valid token: ceil(ctx_len / P)."""
    ctx = np.asarray(ctx_len, dtype=np.int64)
    return (ctx + block_tokens - 1) // block_tokens


# ----------------------------------------------------- a1: block summaries
def block_summaries(keys: np.ndarray, ctx_len: np.ndarray):
    """Per-block, per-channel key min and max over the valid tokens.

    [OasisKV] Figure 7 (left): the GPU keeps "compressed keys" obtained by
    per-block min/max pooling of the full key cache.

    keys: float64 [B, Hkv, N, P, D].  Returns (kmin, kmax), float64
    [B, Hkv, N, D]; a block with no valid token is NaN (never scored).
    """
    B, H, N, P, D = keys.shape
    kmin = np.full((B, H, N, D), np.nan)
    kmax = np.full((B, H, N, D), np.nan)
    for b in range(B):
        ctx = int(ctx_len[b])
        for n in range(int(n_valid_blocks([ctx], P)[0])):
            valid = min(P, ctx - n * P)
            tokens = keys[b, :, n, :valid, :]            # [H, valid, D]
            kmin[b, :, n, :] = tokens.min(axis=1)
            kmax[b, :, n, :] = tokens.max(axis=1)
    return kmin, kmax


def summary_append(kmin, kmax, k_new, ctx_len_before, block_tokens):
    """Fold one appended key row per (b, h) into the summaries, in place.

    The new token sits at position ``ctx_len_before[b]``.  If it opens a new
    block the block's summary becomes that row; otherwise the running
    min/max absorb it.  Summaries "kept up to date on append" is the
    maintenance the compressed-key cache of [OasisKV] Figure 7 needs while
    decoding grows the context; the test suite checks that the result equals
    ``block_summaries`` of the grown context.

    k_new: float64 [B, Hkv, D].
    """
    B = k_new.shape[0]
    for b in range(B):
        pos = int(ctx_len_before[b])
        n, t = divmod(pos, block_tokens)
        if t == 0:
            kmin[b, :, n, :] = k_new[b]
            kmax[b, :, n, :] = k_new[b]
        else:
            kmin[b, :, n, :] = np.minimum(kmin[b, :, n, :], k_new[b])
            kmax[b, :, n, :] = np.maximum(kmax[b, :, n, :], k_new[b])
    return kmin, kmax


def append_token(keys, values, kmin, kmax, pool_k, pool_v, slot_table, ctx_len, k_new, v_new):
    """Write one new token per sequence (R9), in place, and return the grown
    context lengths.

    The row goes to position ``ctx_len[b]`` of every KV head's host keys and
    values, into the summaries (``summary_append``: the compressed keys of
    [OasisKV] Figure 7 stay current while decoding grows the context), and
    into the pool slot holding its block when that block is resident
    ([OasisKV] Figure 9: the slot table names the CPU block each GPU slot
    holds), so that the resident copy keeps matching the host copy.

    keys/values: float64 [B, Hkv, N, P, D]; pool_k/pool_v: float64
    [B, Hkv, K, P, D]; slot_table int [B, Hkv, K]; k_new/v_new: float64
    [B, Hkv, D].
    """
    B, H, N, P, D = keys.shape
    for b in range(B):
        pos = int(ctx_len[b])
        if pos >= N * P:
            raise ValueError(f"sequence {b} is full ({N * P} tokens)")
        n, t = divmod(pos, P)
        keys[b, :, n, t] = k_new[b]
        values[b, :, n, t] = v_new[b]
        for h in range(H):
            for slot in range(slot_table.shape[2]):
                if int(slot_table[b, h, slot]) == n:
                    pool_k[b, h, slot, t] = k_new[b, h]
                    pool_v[b, h, slot, t] = v_new[b, h]
    summary_append(kmin, kmax, k_new, ctx_len, P)
    return np.asarray(ctx_len, dtype=np.int64) + 1


# --------------------------------------------------- a2: lookahead scores
def lookahead_scores(q, kmin, kmax, ctx_len, block_tokens, rows=None):
    """Score every valid block of every (sequence, KV head) with the drafts.

    [OasisKV] Figure 7 (right): the draft query is run against the min/max
    compressed keys, and its result ranks the blocks for the next step;
    method sketch item 2: draft tokens rank the KV blocks the next step will
    need.  The bound is
    Quest's: for one query q and one block, sum over channels of the larger
    of q_c*kmin_c and q_c*kmax_c, an upper bound on q.k for every key of the
    block.  The block's score is the largest bound over the draft rows and
    the G query heads sharing the KV head.

    q: float64 [B, Qn, Hq, D]; kmin/kmax float64 [B, Hkv, N, D].
    rows: the query rows scored (default: the drafts 1..Qn-1, or row 0 when
    Qn == 1); [0] scores with the verification query alone (R16).
    Returns float32 [B, Hkv, N]; blocks at or beyond n_valid are -inf.
    """
    B, Qn, Hq, D = q.shape
    _, H, N, _ = kmin.shape
    G = Hq // H
    if rows is None:
        rows = list(range(1, Qn)) if Qn > 1 else [0]
    nv = n_valid_blocks(ctx_len, block_tokens)
    out = np.full((B, H, N), -np.inf, dtype=np.float32)
    for b in range(B):
        for h in range(H):
            qs = q[b][rows][:, h * G:(h + 1) * G, :].reshape(-1, D)   # [R, D]
            n_b = int(nv[b])
            for n0 in range(0, n_b, 256):
                n1 = min(n_b, n0 + 256)
                lo = kmin[b, h, n0:n1, :]                           # [n, D]
                hi = kmax[b, h, n0:n1, :]
                term = np.maximum(qs[:, None, :] * lo[None], qs[:, None, :] * hi[None])
                bound = term.sum(axis=2)                             # [R, n], fp64
                out[b, h, n0:n1] = bound.max(axis=0).astype(np.float32)
    return out


# ------------------------------------------------------- a3: top-K select
def select_topk(scores, ctx_len, budget_blocks, block_tokens):
    """Per (sequence, KV head): the K best blocks under the token budget.

    [OasisKV] Figure 7: the ranking yields the K blocks the next step uses;
    "What they did" item 4: a 2,048-token KV budget, i.e. K = budget / P
    blocks.
    Ranking: fp32 score descending, ties to the lower block index (R2).  If
    a sequence has no more than K valid blocks, all of them are selected.

    Returns sel int32 [B, Hkv, K] in rank order padded with -1, and the
    matching fp32 scores padded with -inf.
    """
    B, H, N = scores.shape
    K = budget_blocks
    nv = n_valid_blocks(ctx_len, block_tokens)
    sel = np.full((B, H, K), -1, dtype=np.int32)
    sel_score = np.full((B, H, K), -np.inf, dtype=np.float32)
    for b in range(B):
        n_b = int(nv[b])
        idx = np.arange(n_b)
        for h in range(H):
            s = scores[b, h, :n_b].astype(np.float32)
            # Python's sort compares -0.0 and +0.0 as equal, then by index.
            order = sorted(idx.tolist(), key=lambda n: (-float(s[n]), n))
            take = order[:K]
            sel[b, h, :len(take)] = take
            sel_score[b, h, :len(take)] = s[take]
    return sel, sel_score


# ------------------------------------------ a4: residency diff + fetch plan
def plan_fetch(sel, slot_table, last_used, step, fetch_cap, scores=None):
    """Compare the selection with the resident set and plan a capped fetch.

    [OasisKV] method sketch item 3: the prediction is diffed against what is
    already resident on the GPU, only the difference crosses PCIe, and a
    per-step cap keeps that transfer within the link's budget; "What they did" item 3 and
    "Terms in this paper" (capped eviction); Table 2 (LRU eviction);
    Figure 9 (a per-KV-head table mapping each GPU block slot to a CPU
    block).

    Per (b, h), with S* the selected blocks in rank order:
      1. every slot holding a block of S* is stamped last_used = step;
      2. M = blocks of S* not resident, in rank order; F = first min(C, |M|);
      3. victims: free slots ascending, then slots whose block is not in S*
         by (last_used, block id) ascending (R4) - or, when ``scores``
         (float32 [B, Hkv, N], this step's lookahead scores) is given, by
         (score of the block, block id) ascending (R17);
      4. F[i] goes to victims[i], which is stamped last_used = step.

    Inputs are not modified.  Returns a dict with the new slot_table and
    last_used, fetch_slot / fetch_block int32 [B, Hkv, C] (-1 padded) and
    n_fetch int32 [B, Hkv].
    """
    B, H, K = slot_table.shape
    C = fetch_cap
    st = slot_table.copy()
    lu = last_used.copy()
    fetch_slot = np.full((B, H, C), -1, dtype=np.int32)
    fetch_block = np.full((B, H, C), -1, dtype=np.int32)
    n_fetch = np.zeros((B, H), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            selected = [int(x) for x in sel[b, h] if x >= 0]
            assert len(set(selected)) == len(selected), "duplicate selection"
            resident = {}
            for slot in range(K):
                blk = int(st[b, h, slot])
                if blk >= 0:
                    assert blk not in resident, "block resident twice"
                    resident[blk] = slot
            in_sel = set(selected)
            for blk in selected:
                if blk in resident:
                    lu[b, h, resident[blk]] = step
            missing = [blk for blk in selected if blk not in resident]
            fetch = missing[:min(C, len(missing))]
            free = [slot for slot in range(K) if st[b, h, slot] < 0]
            stale = [slot for slot in range(K)
                     if st[b, h, slot] >= 0 and int(st[b, h, slot]) not in in_sel]
            if scores is None:
                stale.sort(key=lambda slot: (int(lu[b, h, slot]), int(st[b, h, slot])))
            else:
                stale.sort(key=lambda slot: (float(scores[b, h, st[b, h, slot]]), int(st[b, h, slot])))
            victims = free + stale
            assert len(victims) >= len(fetch)
            for i, blk in enumerate(fetch):
                slot = victims[i]
                st[b, h, slot] = blk
                lu[b, h, slot] = step
                fetch_slot[b, h, i] = slot
                fetch_block[b, h, i] = blk
            n_fetch[b, h] = len(fetch)
    return {"slot_table": st, "last_used": lu, "fetch_slot": fetch_slot,
            "fetch_block": fetch_block, "n_fetch": n_fetch}


# ------------------------------------------------------- a5: H2D gather
def prefetch(host_kv, pool, fetch_slot, fetch_block, n_fetch):
    """Copy each planned block from the host KV cache into its pool slot.

    [OasisKV] Figure 7: the chosen blocks come in from the CPU-side KV cache
    ahead of use; Figure 8: the copy completes before the same layer attends
    at step t+1.
    host_kv: [B, Hkv, N, ...]; pool: [B, Hkv, K, ...] (same trailing shape,
    any dtype: the copy is bytewise).  Returns a new pool array.
    """
    out = pool.copy()
    B, H = n_fetch.shape
    for b in range(B):
        for h in range(H):
            for i in range(int(n_fetch[b, h])):
                out[b, h, int(fetch_slot[b, h, i])] = host_kv[b, h, int(fetch_block[b, h, i])]
    return out


# ------------------------------------------------ a6: sparse GQA attention
def sparse_attention(q, pool_k, pool_v, slot_table, ctx_len, scale):
    """GQA decode attention of all Qn query rows over the resident blocks.

    [OasisKV] Figure 7 (right): the verification query and the drafts are
    attended in one pass over the resident sparse working set; Figure 9:
    slot table entries name the CPU block each GPU slot holds.

    q: float64 [B, Qn, Hq, D]; pool_k / pool_v: float64 [B, Hkv, K, P, D];
    slot_table int32 [B, Hkv, K].  Returns o float64 [B, Qn, Hq, D] and
    lse float64 [B, Qn, Hq] (natural log of the sum of exp(scale*q.k)).
    """
    B, Qn, Hq, D = q.shape
    _, H, K, P, _ = pool_k.shape
    G = Hq // H
    o = np.zeros((B, Qn, Hq, D))
    lse = np.full((B, Qn, Hq), -np.inf)
    for b in range(B):
        ctx = int(ctx_len[b])
        for h in range(H):
            ks, vs = [], []
            for slot in range(K):
                blk = int(slot_table[b, h, slot])
                if blk < 0:
                    continue
                valid = min(P, ctx - blk * P)
                if valid <= 0:
                    continue
                ks.append(pool_k[b, h, slot, :valid])
                vs.append(pool_v[b, h, slot, :valid])
            if not ks:
                continue                                   # R6
            kt = np.concatenate(ks)                        # [T, D]
            vt = np.concatenate(vs)
            qh = q[b, :, h * G:(h + 1) * G, :].reshape(-1, D)   # rows (j, g)
            logits = scale * (qh @ kt.T)                   # [Qn*G, T]
            m = logits.max(axis=1, keepdims=True)
            p = np.exp(logits - m)
            l = p.sum(axis=1, keepdims=True)
            o[b, :, h * G:(h + 1) * G, :] = ((p @ vt) / l).reshape(Qn, G, D)
            lse[b, :, h * G:(h + 1) * G] = (m + np.log(l)).reshape(Qn, G)
    return o, lse


def dense_attention(q, keys, values, ctx_len, scale):
    """Full attention over every valid context token (the "Full" anchor of
    [OasisKV] Table 1): the special case the sparse path must reproduce when
    the budget covers the whole context.  keys/values [B, Hkv, N, P, D]."""
    B, Qn, Hq, D = q.shape
    _, H, N, P, _ = keys.shape
    G = Hq // H
    o = np.zeros((B, Qn, Hq, D))
    lse = np.full((B, Qn, Hq), -np.inf)
    for b in range(B):
        ctx = int(ctx_len[b])
        if ctx == 0:
            continue
        for h in range(H):
            kt = keys[b, h].reshape(N * P, D)[:ctx]
            vt = values[b, h].reshape(N * P, D)[:ctx]
            qh = q[b, :, h * G:(h + 1) * G, :].reshape(-1, D)
            logits = scale * (qh @ kt.T)
            m = logits.max(axis=1, keepdims=True)
            p = np.exp(logits - m)
            l = p.sum(axis=1, keepdims=True)
            o[b, :, h * G:(h + 1) * G, :] = ((p @ vt) / l).reshape(Qn, G, D)
            lse[b, :, h * G:(h + 1) * G] = (m + np.log(l)).reshape(Qn, G)
    return o, lse


# ------------------------------------ prediction quality (R16): set overlap
def block_overlap(a, b):
    """Per (sequence, KV head): how many distinct block ids of list ``b`` also
    occur in list ``a`` (-1 entries are empty).  a, b: int [B, Hkv, *]."""
    B, H = a.shape[:2]
    out = np.zeros((B, H), dtype=np.int32)
    for i in range(B):
        for h in range(H):
            sa = {int(x) for x in a[i, h] if x >= 0}
            sb = {int(x) for x in b[i, h] if x >= 0}
            out[i, h] = len(sa & sb)
    return out


# ---------------------------------------------- residency loss (R19)
def evict_slots(slot_table, mask):
    """Frees every slot whose mask entry is set (R19).  Returns a new table."""
    st = slot_table.copy()
    st[np.asarray(mask, dtype=bool)] = -1
    return st


# ------------------------------------------------ a7: per-step order
def decode_layer_steps(keys, values, kmin, kmax, ctx_len, q_prime, q_steps,
                       budget_blocks, fetch_cap, scale, host_kv_bits=None, corrective=False,
                       evict_masks=None, appends=None):
    """One layer through priming and T decode steps, in the pages' order.

    [OasisKV] Figure 8: at step t the drafts drive the top-K prediction,
    the selection and the copy, and all of it completes before the same
    layer attends at step t+1; Figure 7 (right): attention at step t runs over the working set
    staged by step t-1.  Priming (a cold pool) runs one
    select / plan / fetch from ``q_prime`` at step 0; decode step t
    (t = 1..T) runs attention over the working set, then select / plan /
    fetch from that step's drafts.

    keys/values: float64 [B, Hkv, N, P, D]; q_prime, q_steps[t]: float64
    [B, Qn, Hq, D].  Returns a list of per-step dicts (attention output,
    selection, plan) plus the final slot table.

    With ``corrective`` each decode step first finds the exact set E_t from
    the verification row, records the agreement counts of the lookahead and
    previous-token predictions and the resident coverage of E_t, and fetches
    E_t's missing blocks without a cap before the attention (R16).
    ``evict_masks[t-1]`` (bool [B, Hkv, K]), when given, frees slots after the
    attention of decode step t and before its plan (R19).
    ``appends[t-1]`` = (k_new, v_new), float64 [B, Hkv, D], when given, is the
    token written at the start of decode step t, before anything else of that
    step (R9); the caller's arrays are left as they were (the grown keys,
    values and summaries are copies) and each record carries the context
    length its step used as ``ctx_len``.
    """
    B, H, N, P, D = keys.shape
    if appends is not None:
        keys, values, kmin, kmax = keys.copy(), values.copy(), kmin.copy(), kmax.copy()
    ctx_len = np.asarray(ctx_len, dtype=np.int64).copy()
    K = budget_blocks
    st = np.full((B, H, K), -1, dtype=np.int32)
    lu = np.full((B, H, K), -1, dtype=np.int32)
    pool_k = np.zeros((B, H, K, P, D))
    pool_v = np.zeros((B, H, K, P, D))
    records = []

    def select_plan_fetch(qs, step):
        nonlocal st, lu, pool_k, pool_v
        sc = lookahead_scores(qs, kmin, kmax, ctx_len, P)
        sel, sel_score = select_topk(sc, ctx_len, K, P)
        plan = plan_fetch(sel, st, lu, step, fetch_cap)
        pool_k = prefetch(keys, pool_k, plan["fetch_slot"], plan["fetch_block"], plan["n_fetch"])
        pool_v = prefetch(values, pool_v, plan["fetch_slot"], plan["fetch_block"], plan["n_fetch"])
        st, lu = plan["slot_table"], plan["last_used"]
        return sc, sel, sel_score, plan

    def corrective_fetch(qs, step, sel_lookahead, exact_prev):
        nonlocal st, lu, pool_k, pool_v
        exact, _ = select_topk(lookahead_scores(qs, kmin, kmax, ctx_len, P, rows=[0]), ctx_len, K, P)
        rec = {"exact": exact,
               "agree_lookahead": block_overlap(sel_lookahead, exact),
               "agree_prev": block_overlap(exact_prev, exact) if exact_prev is not None else None,
               "covered": block_overlap(st, exact)}
        plan = plan_fetch(exact, st, lu, step, K)
        pool_k = prefetch(keys, pool_k, plan["fetch_slot"], plan["fetch_block"], plan["n_fetch"])
        pool_v = prefetch(values, pool_v, plan["fetch_slot"], plan["fetch_block"], plan["n_fetch"])
        st, lu = plan["slot_table"], plan["last_used"]
        rec["plan"] = plan
        return rec

    _, sel_prev, _, _ = select_plan_fetch(q_prime, 0)
    exact_prev = None
    for t, qs in enumerate(q_steps, start=1):
        if appends is not None:
            k_new, v_new = appends[t - 1]
            ctx_len = append_token(keys, values, kmin, kmax, pool_k, pool_v, st, ctx_len, k_new, v_new)
        corr = None
        if corrective:
            corr = corrective_fetch(qs, t, sel_prev, exact_prev)
            exact_prev = corr["exact"]
        o, lse = sparse_attention(qs, pool_k, pool_v, st, ctx_len, scale)
        slot_table_used = st.copy()
        if evict_masks is not None:
            st = evict_slots(st, evict_masks[t - 1])
        sc, sel, sel_score, plan = select_plan_fetch(qs, t)
        sel_prev = sel
        records.append({"o": o, "lse": lse, "slot_table_attn": slot_table_used,
                        "scores": sc, "sel": sel, "sel_score": sel_score, "plan": plan,
                        "corrective": corr, "ctx_len": ctx_len.copy()})
    return records, st, lu


def default_scale(head_dim: int) -> float:
    """Softmax scale 1/sqrt(D) of standard dot-product attention."""
    return 1.0 / math.sqrt(head_dim)
