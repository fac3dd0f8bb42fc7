"""Pins for the CPU oracle, checked against facts that do not come from the
oracle itself: hand-worked examples from the pages' definitions, closed forms,
bounds that must hold, brute force, and library routines for the special cases
the method reduces to.  CPU only."""

import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


def _bf16_round(x):
    """Round float64 values to bf16-representable values (test input prep)."""
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).double().numpy()


# ------------------------------------------------------------ summaries
def test_summaries_hand_worked():
    # P = 4, D = 2, one head, ctx 6: block 0 full, block 1 has 2 valid tokens.
    keys = np.zeros((1, 1, 3, 4, 2))
    keys[0, 0, 0] = [[1, -1], [3, 2], [-2, 0], [0.5, 5]]
    keys[0, 0, 1] = [[7, 7], [-7, 1], [100, -100], [100, -100]]   # last two masked
    keys[0, 0, 2] = 42.0                                          # no valid token
    kmin, kmax = O.block_summaries(keys, np.array([6]))
    assert kmin[0, 0, 0].tolist() == [-2, -1] and kmax[0, 0, 0].tolist() == [3, 5]
    assert kmin[0, 0, 1].tolist() == [-7, 1] and kmax[0, 0, 1].tolist() == [7, 7]
    assert np.isnan(kmin[0, 0, 2]).all() and np.isnan(kmax[0, 0, 2]).all()


def test_summaries_bound_and_attained():
    r = _rng(1)
    B, H, N, P, D = 2, 3, 5, 16, 8
    keys = _bf16_round(r.standard_normal((B, H, N, P, D)))
    ctx = np.array([70, 33])
    kmin, kmax = O.block_summaries(keys, ctx)
    for b in range(B):
        for n in range(N):
            valid = min(P, ctx[b] - n * P)
            if valid <= 0:
                assert np.isnan(kmin[b, :, n]).all()
                continue
            tok = keys[b, :, n, :valid]                       # [H, valid, D]
            assert (tok >= kmin[b, :, n][:, None]).all() and (tok <= kmax[b, :, n][:, None]).all()
            assert (tok == kmin[b, :, n][:, None]).any(axis=1).all()
            assert (tok == kmax[b, :, n][:, None]).any(axis=1).all()


def test_summaries_ignore_masked_tokens():
    r = _rng(2)
    keys = _bf16_round(r.standard_normal((1, 2, 4, 16, 4)))
    ctx = np.array([40])
    a = O.block_summaries(keys, ctx)
    keys2 = keys.copy()
    keys2[0, :, 2, 8:] = 1e6         # tokens 40..47 are beyond the context
    keys2[0, :, 3] = -1e6
    b = O.block_summaries(keys2, ctx)
    np.testing.assert_array_equal(a[0][:, :, :3], b[0][:, :, :3])
    np.testing.assert_array_equal(a[1][:, :, :3], b[1][:, :, :3])


def test_summary_append_equals_rebuild():
    r = _rng(3)
    B, H, N, P, D = 3, 2, 4, 16, 8
    keys = _bf16_round(r.standard_normal((B, H, N, P, D)))
    ctx = np.array([15, 16, 47])          # append lands at t=15, t=0 (new block), t=15
    kmin, kmax = O.block_summaries(keys, ctx)
    k_new = _bf16_round(r.standard_normal((B, H, D)) * 3)
    O.summary_append(kmin, kmax, k_new, ctx, P)
    grown = keys.copy()
    for b in range(B):
        n, t = divmod(int(ctx[b]), P)
        grown[b, :, n, t] = k_new[b]
    kmin2, kmax2 = O.block_summaries(grown, ctx + 1)
    np.testing.assert_array_equal(kmin, kmin2)
    np.testing.assert_array_equal(kmax, kmax2)


# ---------------------------------------------------------------- scores
def _read_score_golden():
    keys, queries, expect, selects = {}, {}, None, []
    with open(os.path.join(GOLDEN, "score_tiny.txt")) as f:
        for line in f:
            line = line.split("#")[0].split()
            if not line:
                continue
            if line[0] == "key":
                keys[int(line[1])] = [float(v) for v in line[2:]]
            elif line[0] == "query":
                queries[(int(line[1]), int(line[2]))] = [float(v) for v in line[3:]]
            elif line[0] == "score":
                expect = [float(v) for v in line[1:]]
            elif line[0] == "select":
                selects.append((int(line[1]), [int(v) for v in line[2:]]))
    return keys, queries, expect, selects


def test_scores_hand_worked_golden():
    keys, queries, expect, selects = _read_score_golden()
    P, D = 2, 2
    kb = np.array([keys[i] for i in range(6)]).reshape(1, 1, 3, P, D)
    q = np.zeros((1, 2, 2, D))
    for (j, h), v in queries.items():
        q[0, j, h] = v
    ctx = np.array([5])
    kmin, kmax = O.block_summaries(kb, ctx)
    s = O.lookahead_scores(q, kmin, kmax, ctx, P)
    assert s[0, 0].tolist() == expect
    for k, want in selects:
        sel, _ = O.select_topk(s, ctx, k, P)
        assert sel[0, 0].tolist() == want


def test_scores_upper_bound_brute_force():
    r = _rng(4)
    B, Qn, Hq, H, N, P, D = 2, 4, 6, 2, 6, 16, 16
    keys = _bf16_round(r.standard_normal((B, H, N, P, D)))
    q = _bf16_round(r.standard_normal((B, Qn, Hq, D)))
    ctx = np.array([96, 57])
    kmin, kmax = O.block_summaries(keys, ctx)
    s = O.lookahead_scores(q, kmin, kmax, ctx, P)
    G = Hq // H
    for b in range(B):
        for h in range(H):
            drafts = q[b, 1:, h * G:(h + 1) * G].reshape(-1, D)
            for n in range(N):
                valid = min(P, ctx[b] - n * P)
                if valid <= 0:
                    assert s[b, h, n] == -np.inf
                    continue
                best = (drafts @ keys[b, h, n, :valid].T).max()
                assert s[b, h, n] >= np.float32(best) - 1e-4 * abs(best)


def test_scores_reduce_to_dot_product_when_block_is_one_token():
    # P = 1: kmin = kmax = k, so the bound is exactly max_{drafts, group} q.k,
    # a plain matrix product.
    r = _rng(5)
    B, Qn, Hq, H, N, D = 1, 3, 4, 2, 9, 32
    keys = _bf16_round(r.standard_normal((B, H, N, 1, D)))
    q = _bf16_round(r.standard_normal((B, Qn, Hq, D)))
    ctx = np.array([N])
    kmin, kmax = O.block_summaries(keys, ctx)
    s = O.lookahead_scores(q, kmin, kmax, ctx, 1)
    G = Hq // H
    for h in range(H):
        drafts = q[0, 1:, h * G:(h + 1) * G].reshape(-1, D)
        ref = torch.from_numpy(drafts) @ torch.from_numpy(keys[0, h, :, 0]).T   # fp64 matmul
        want = ref.max(dim=0).values.numpy().astype(np.float32)
        np.testing.assert_allclose(s[0, h], want, rtol=1e-7, atol=0)


def test_scores_identical_tokens_are_tight():
    # A block whose tokens are all equal has kmin = kmax = k: the bound is q.k.
    r = _rng(6)
    D = 8
    k = _bf16_round(r.standard_normal(D))
    keys = np.broadcast_to(k, (1, 1, 1, 16, D)).copy()
    q = _bf16_round(r.standard_normal((1, 2, 1, D)))
    kmin, kmax = O.block_summaries(keys, np.array([16]))
    s = O.lookahead_scores(q, kmin, kmax, np.array([16]), 16)
    assert s[0, 0, 0] == np.float32(q[0, 1, 0] @ k)


def test_scores_ignore_verification_row_and_scale_linearly():
    r = _rng(7)
    B, Qn, Hq, H, N, P, D = 1, 3, 4, 2, 5, 16, 8
    keys = _bf16_round(r.standard_normal((B, H, N, P, D)))
    q = _bf16_round(r.standard_normal((B, Qn, Hq, D)))
    ctx = np.array([N * P])
    kmin, kmax = O.block_summaries(keys, ctx)
    s = O.lookahead_scores(q, kmin, kmax, ctx, P)
    q2 = q.copy()
    q2[:, 0] = 1e3
    np.testing.assert_array_equal(s, O.lookahead_scores(q2, kmin, kmax, ctx, P))
    q3 = q.copy()
    q3[:, 2] *= -1.0                          # a draft row changes -> scores change
    assert not np.array_equal(s, O.lookahead_scores(q3, kmin, kmax, ctx, P))
    # positive homogeneity: the bound has no constant term
    np.testing.assert_allclose(O.lookahead_scores(2 * q, kmin, kmax, ctx, P), 2 * s, rtol=1e-7)


def test_scores_single_query_row_uses_row_zero():
    r = _rng(8)
    keys = _bf16_round(r.standard_normal((1, 1, 3, 16, 8)))
    q = _bf16_round(r.standard_normal((1, 1, 2, 8)))
    ctx = np.array([48])
    kmin, kmax = O.block_summaries(keys, ctx)
    s1 = O.lookahead_scores(q, kmin, kmax, ctx, 16)
    q2 = np.concatenate([np.zeros_like(q), q], axis=1)   # same row as a draft
    np.testing.assert_array_equal(s1, O.lookahead_scores(q2, kmin, kmax, ctx, 16))


# ---------------------------------------------------------------- select
def _naive_topk(s, k):
    """Repeated arg-max: take the largest remaining score, lowest index on ties."""
    s = [float(x) for x in s]
    taken, out = set(), []
    for _ in range(min(k, len(s))):
        best = None
        for i, v in enumerate(s):
            if i in taken:
                continue
            if best is None or v > s[best]:
                best = i
        taken.add(best)
        out.append(best)
    return out


@pytest.mark.parametrize("seed", range(5))
def test_select_matches_repeated_argmax(seed):
    r = _rng(10 + seed)
    N, K = 50, 12
    s = r.integers(-4, 5, size=(1, 2, N)).astype(np.float32)   # many exact ties
    s[0, 1, ::7] = -0.0
    s[0, 1, 3::7] = 0.0
    ctx = np.array([N * 16 - 5])
    sel, sc = O.select_topk(s, ctx, K, 16)
    for h in range(2):
        assert sel[0, h].tolist() == _naive_topk(s[0, h], K)
        np.testing.assert_array_equal(sc[0, h], s[0, h][sel[0, h]])


def test_select_takes_all_when_context_fits_budget():
    s = np.array([[[3.0, 1.0, 2.0, 9.0, 9.0, -np.inf]]], dtype=np.float32)
    sel, sc = O.select_topk(s, np.array([5 * 16 - 3]), 8, 16)
    assert sel[0, 0].tolist() == [3, 4, 0, 2, 1, -1, -1, -1]
    assert sc[0, 0, 5] == -np.inf


# ------------------------------------------------------------------ plan
def _read_plan_golden():
    rows = []
    with open(os.path.join(GOLDEN, "plan_tiny.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            cols = [c.split() for c in line.split("|")]
            to_ints = lambda c: [] if c == ["-"] else [int(v) for v in c]
            rows.append(tuple(to_ints(c) for c in cols))
    return rows


def test_plan_hand_worked_golden():
    st = np.full((1, 1, 3), -1, dtype=np.int32)
    lu = np.full((1, 1, 3), -1, dtype=np.int32)
    for (step,), (cap,), sel, st_after, lu_after, f_slot, f_block in _read_plan_golden():
        plan = O.plan_fetch(np.array([[sel]], dtype=np.int32), st, lu, step, cap)
        assert plan["slot_table"][0, 0].tolist() == st_after, step
        assert plan["last_used"][0, 0].tolist() == lu_after, step
        n = int(plan["n_fetch"][0, 0])
        assert plan["fetch_slot"][0, 0, :n].tolist() == f_slot, step
        assert plan["fetch_block"][0, 0, :n].tolist() == f_block, step
        assert (plan["fetch_slot"][0, 0, n:] == -1).all()
        st, lu = plan["slot_table"], plan["last_used"]


def test_plan_invariants_random_sequences():
    r = _rng(20)
    B, H, N, K, C = 2, 3, 40, 8, 3
    st = np.full((B, H, K), -1, dtype=np.int32)
    lu = np.full((B, H, K), -1, dtype=np.int32)
    for step in range(60):
        sel = np.full((B, H, K), -1, dtype=np.int32)
        for b in range(B):
            for h in range(H):
                m = r.integers(1, K + 1)
                sel[b, h, :m] = r.choice(N, size=m, replace=False)
        plan = O.plan_fetch(sel, st, lu, step, C)
        for b in range(B):
            for h in range(H):
                before = [x for x in st[b, h] if x >= 0]
                after = [x for x in plan["slot_table"][b, h] if x >= 0]
                chosen = [x for x in sel[b, h] if x >= 0]
                missing = [x for x in chosen if x not in before]
                n = plan["n_fetch"][b, h]
                fetched = plan["fetch_block"][b, h, :n].tolist()
                assert len(after) <= K and len(set(after)) == len(after)
                assert n == min(C, len(missing)) and fetched == missing[:n]
                assert all(x not in before for x in fetched)
                assert all(x in after for x in chosen if x in before)     # hits never evicted
                assert set(after) <= set(before) | set(fetched)
                for slot in range(K):
                    blk = plan["slot_table"][b, h, slot]
                    if blk in chosen:
                        assert plan["last_used"][b, h, slot] == step
                # evicted blocks were the least recently used stale ones
                evicted = set(before) - set(after)
                kept_stale = [x for x in set(before) & set(after) if x not in chosen]
                if evicted and kept_stale:
                    age = {int(st[b, h, s]): (int(lu[b, h, s]), int(st[b, h, s]))
                           for s in range(K) if st[b, h, s] >= 0}
                    assert max(age[x] for x in evicted) < min(age[x] for x in kept_stale)
        st, lu = plan["slot_table"], plan["last_used"]


# --------------------------------------------------------------- prefetch
def test_prefetch_copies_only_planned_slots():
    r = _rng(30)
    host = r.integers(0, 65535, size=(1, 2, 10, 2, 16, 4)).astype(np.uint16)
    pool = np.zeros((1, 2, 4, 2, 16, 4), dtype=np.uint16)
    fs = np.array([[[2, 0, -1], [3, -1, -1]]], dtype=np.int32)
    fb = np.array([[[7, 1, -1], [9, -1, -1]]], dtype=np.int32)
    nf = np.array([[2, 1]], dtype=np.int32)
    out = O.prefetch(host, pool, fs, fb, nf)
    assert (out[0, 0, 2] == host[0, 0, 7]).all() and (out[0, 0, 0] == host[0, 0, 1]).all()
    assert (out[0, 1, 3] == host[0, 1, 9]).all()
    assert (out[0, 0, [1, 3]] == 0).all() and (out[0, 1, :3] == 0).all()


# -------------------------------------------------------------- attention
def test_attention_hand_worked_two_tokens():
    # logits 0 and ln 3 -> weights 1/4, 3/4.
    P, D = 2, 2
    pk = np.zeros((1, 1, 1, P, D)); pv = np.zeros((1, 1, 1, P, D))
    pk[0, 0, 0, 1] = [math.log(3.0), 0.0]
    pv[0, 0, 0, 0] = [1.0, 0.0]; pv[0, 0, 0, 1] = [0.0, 2.0]
    q = np.array([[[[1.0, 0.0]]]])
    o, lse = O.sparse_attention(q, pk, pv, np.array([[[0]]], dtype=np.int32), np.array([2]), 1.0)
    np.testing.assert_allclose(o[0, 0, 0], [0.25, 1.5], rtol=1e-14)
    np.testing.assert_allclose(lse[0, 0, 0], math.log(4.0), rtol=1e-14)


def test_attention_single_token_and_empty():
    r = _rng(31)
    P, D = 16, 8
    pk = r.standard_normal((1, 2, 2, P, D)); pv = r.standard_normal((1, 2, 2, P, D))
    q = r.standard_normal((1, 2, 4, D))
    st = np.array([[[3, -1], [-1, -1]]], dtype=np.int32)
    ctx = np.array([3 * P + 1])                   # block 3 holds exactly one valid token
    o, lse = O.sparse_attention(q, pk, pv, st, ctx, 0.3)
    for j in range(2):
        for g in range(2):
            np.testing.assert_allclose(o[0, j, g], pv[0, 0, 0, 0], rtol=1e-14)
            np.testing.assert_allclose(lse[0, j, g], 0.3 * q[0, j, g] @ pk[0, 0, 0, 0], rtol=1e-13)
    assert (o[0, :, 2:] == 0).all() and (lse[0, :, 2:] == -np.inf).all()


def test_attention_budget_covering_context_equals_dense_sdpa():
    """With every block resident (in a shuffled slot order), sparse attention
    is dense attention, checked against torch's scaled_dot_product_attention."""
    r = _rng(32)
    B, Qn, Hq, H, N, P, D = 2, 3, 8, 2, 5, 16, 16
    keys = r.standard_normal((B, H, N, P, D)); vals = r.standard_normal((B, H, N, P, D))
    q = r.standard_normal((B, Qn, Hq, D))
    ctx = np.array([N * P, 2 * P + 5])
    K = 7
    st = np.full((B, H, K), -1, dtype=np.int32)
    pk = np.zeros((B, H, K, P, D)); pv = np.zeros((B, H, K, P, D))
    for b in range(B):
        for h in range(H):
            slots = r.permutation(K)[:N]
            for n, s in enumerate(slots):
                st[b, h, s] = n
                pk[b, h, s] = keys[b, h, n]; pv[b, h, s] = vals[b, h, n]
    scale = 1 / math.sqrt(D)
    o, lse = O.sparse_attention(q, pk, pv, st, ctx, scale)
    G = Hq // H
    for b in range(B):
        L = int(ctx[b])
        kt = torch.from_numpy(keys[b].reshape(H, N * P, D)[:, :L])       # [H, L, D]
        vt = torch.from_numpy(vals[b].reshape(H, N * P, D)[:, :L])
        qt = torch.from_numpy(q[b]).permute(1, 0, 2)                      # [Hq, Qn, D]
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt, kt.repeat_interleave(G, 0), vt.repeat_interleave(G, 0), scale=scale)
        np.testing.assert_allclose(o[b], ref.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
        ref_lse = torch.logsumexp(scale * qt @ kt.repeat_interleave(G, 0).transpose(1, 2), dim=-1)
        np.testing.assert_allclose(lse[b], ref_lse.T.numpy(), rtol=1e-12)
    # dense_attention is the same anchor
    od, lsed = O.dense_attention(q, keys, vals, ctx, scale)
    np.testing.assert_allclose(o, od, rtol=1e-10, atol=1e-12)


def test_attention_ignores_masked_tokens():
    r = _rng(33)
    P, D = 16, 8
    pk = r.standard_normal((1, 1, 2, P, D)); pv = r.standard_normal((1, 1, 2, P, D))
    q = r.standard_normal((1, 1, 1, D))
    st = np.array([[[0, 1]]], dtype=np.int32)
    ctx = np.array([P + 9])
    o, lse = O.sparse_attention(q, pk, pv, st, ctx, 0.5)
    pk2, pv2 = pk.copy(), pv.copy()
    pk2[0, 0, 1, 9:] = 50.0; pv2[0, 0, 1, 9:] = 1e9
    o2, lse2 = O.sparse_attention(q, pk2, pv2, st, ctx, 0.5)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)


# ---------------------------------------------------------- whole steps
def test_planted_blocks_are_always_selected():
    """Planted relevant blocks (keys 0.5*u + noise, u the query mean) are
    recalled at priming and at every step of the tiny workload."""
    from lookahead_sparse_kv_b200 import workloads as W
    w = W.WORKLOADS["tiny"]
    kv = O.bf16_bits_to_f64(W.bf16_bits(W.make_host_kv(w)))
    keys = kv[:, :, :, 0]
    ctx = W.initial_ctx_len(w).numpy()
    kmin, kmax = O.block_summaries(keys, ctx)
    qs = W.QueryStream(w)
    planted = W.planted_positions(w, 0)[0].numpy()
    for _ in range(w.steps + 1):
        q = O.bf16_bits_to_f64(W.bf16_bits(qs.next()))
        sel, _ = O.select_topk(O.lookahead_scores(q, kmin, kmax, ctx, 16), ctx, w.budget_blocks, 16)
        for b in range(w.batch):
            for h in range(w.n_kv_heads):
                assert set(planted[b, h].tolist()) <= set(sel[b, h].tolist())


def test_decode_steps_with_full_budget_are_dense():
    """Budget and cap at least the context: after priming every block is
    resident, so each step's attention is dense attention."""
    r = _rng(40)
    B, Qn, Hq, H, N, P, D = 1, 3, 4, 2, 6, 16, 16
    keys = _bf16_round(r.standard_normal((B, H, N, P, D)))
    vals = _bf16_round(r.standard_normal((B, H, N, P, D)))
    ctx = np.array([N * P - 3])
    kmin, kmax = O.block_summaries(keys, ctx)
    qp = _bf16_round(r.standard_normal((B, Qn, Hq, D)))
    qsteps = [_bf16_round(r.standard_normal((B, Qn, Hq, D))) for _ in range(3)]
    recs, st, _ = O.decode_layer_steps(keys, vals, kmin, kmax, ctx, qp, qsteps,
                                       budget_blocks=N, fetch_cap=N, scale=0.25)
    for rec, qs in zip(recs, qsteps):
        od, lsed = O.dense_attention(qs, keys, vals, ctx, 0.25)
        np.testing.assert_allclose(rec["o"], od, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(rec["lse"], lsed, rtol=1e-12)
    assert sorted(st[0, 0].tolist()) == list(range(N))


def test_append_token_writes_host_summary_and_resident_slot():
    """Three appended tokens, the second opening a new block: the host rows
    hold the new values, the summaries equal a rebuild of the grown context,
    the slot that holds the block gets the row and no other slot changes."""
    r = _rng(41)
    B, H, N, P, D, K = 2, 2, 4, 4, 8, 3
    keys = _bf16_round(r.standard_normal((B, H, N, P, D)))
    vals = _bf16_round(r.standard_normal((B, H, N, P, D)))
    ctx = np.array([2 * P - 1, P])                        # one token short of a block / a fresh block
    kmin, kmax = O.block_summaries(keys, ctx)
    st = np.array([[[1, -1, 0], [-1, 2, -1]], [[1, 0, -1], [3, -1, 1]]], dtype=np.int32)
    pool_k = np.zeros((B, H, K, P, D))
    pool_v = np.zeros((B, H, K, P, D))
    for b in range(B):
        for h in range(H):
            for slot in range(K):
                if st[b, h, slot] >= 0:
                    pool_k[b, h, slot] = keys[b, h, st[b, h, slot]]
                    pool_v[b, h, slot] = vals[b, h, st[b, h, slot]]
    k0, v0 = keys.copy(), vals.copy()
    for step in range(3):
        pk_before, pv_before = pool_k.copy(), pool_v.copy()
        k_new = _bf16_round(r.standard_normal((B, H, D)))
        v_new = _bf16_round(r.standard_normal((B, H, D)))
        pos = ctx.copy()
        ctx = O.append_token(keys, vals, kmin, kmax, pool_k, pool_v, st, ctx, k_new, v_new)
        for b in range(B):
            n, t = divmod(int(pos[b]), P)
            k0[b, :, n, t], v0[b, :, n, t] = k_new[b], v_new[b]
            for h in range(H):
                for slot in range(K):
                    if st[b, h, slot] == n:
                        pk_before[b, h, slot, t] = k_new[b, h]
                        pv_before[b, h, slot, t] = v_new[b, h]
        np.testing.assert_array_equal(ctx, pos + 1)
        np.testing.assert_array_equal(keys, k0)
        np.testing.assert_array_equal(vals, v0)
        np.testing.assert_array_equal(pool_k, pk_before)
        np.testing.assert_array_equal(pool_v, pv_before)
        rmin, rmax = O.block_summaries(keys, ctx)
        np.testing.assert_array_equal(kmin, rmin)
        np.testing.assert_array_equal(kmax, rmax)
    # the resident slot of sequence 1's second block got all three rows
    np.testing.assert_array_equal(pool_k[1, 0, 0, :3], keys[1, 0, 1, :3])


def test_decode_steps_with_appends_and_full_budget_are_dense():
    """Full budget with one appended token per step (the context crosses a
    block boundary): each step's attention equals dense attention over the
    grown context, so the new token is visible to the step it was appended
    at and the resident copy of its block stays current.  The one exception
    is a token that opens a new block: that block is not resident yet (the
    step's own plan fetches it, Figure 8), so at that step it is the one
    token dense attention must leave out."""
    r = _rng(42)
    B, Qn, Hq, H, N, P, D = 2, 3, 4, 2, 6, 16, 16
    keys = _bf16_round(r.standard_normal((B, H, N, P, D)))
    vals = _bf16_round(r.standard_normal((B, H, N, P, D)))
    ctx = np.array([4 * P - 2, 5 * P - 1])
    kmin, kmax = O.block_summaries(keys, ctx)
    qp = _bf16_round(r.standard_normal((B, Qn, Hq, D)))
    steps = 5
    qsteps = [_bf16_round(r.standard_normal((B, Qn, Hq, D))) for _ in range(steps)]
    apps = [(_bf16_round(r.standard_normal((B, H, D))), _bf16_round(r.standard_normal((B, H, D))))
            for _ in range(steps)]
    k_in, v_in = keys.copy(), vals.copy()
    recs, st, _ = O.decode_layer_steps(keys, vals, kmin, kmax, ctx, qp, qsteps, budget_blocks=N, fetch_cap=N,
                                       scale=0.25, appends=apps)
    np.testing.assert_array_equal(keys, k_in)               # the caller's arrays are not grown
    grown_k, grown_v, c = keys.copy(), vals.copy(), ctx.copy()
    opened = 0
    for t, (rec, qs) in enumerate(zip(recs, qsteps)):
        visible = c + 1
        for b in range(B):
            n, tok = divmod(int(c[b]), P)
            grown_k[b, :, n, tok] = apps[t][0][b]
            grown_v[b, :, n, tok] = apps[t][1][b]
            if tok == 0:
                visible[b] -= 1
                opened += 1
        c = c + 1
        np.testing.assert_array_equal(rec["ctx_len"], c)
        od, lsed = O.dense_attention(qs, grown_k, grown_v, visible, 0.25)
        np.testing.assert_allclose(rec["o"], od, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(rec["lse"], lsed, rtol=1e-12)
    assert opened == 2                                      # both sequences crossed a block boundary


def test_bf16_widening_matches_torch_on_every_bit_pattern():
    """Every one of the 65,536 bf16 patterns widens to the value torch's own
    bf16 -> float64 conversion gives (NaNs stay NaN); narrowing inverts it
    on the non-NaN patterns and refuses values that would need rounding."""
    import torch
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):                # signalling-NaN patterns
        ours = O.bf16_bits_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))      # -0.0 kept
    back = O.f64_to_bf16_bits(ours[~nan])
    assert np.array_equal(back, bits[~nan])
    for x in (1.0 + 2.0 ** -8, 1.0 / 3.0, 2.0 ** -140 * 1.5):
        with pytest.raises(ValueError):
            O.f64_to_bf16_bits(np.array([x]))
