"""Pins for the oracle's prediction-quality pieces (exact set, set overlap,
corrective fetch) and for the leading-draft query generator.  CPU only.

OasisKV, Figure 4 (top-K prediction accuracy with the previous token vs a
lookahead token) and Figure 6 (agreement of the draft-predicted top-K with the
true next-token top-K); "What they did": prediction misses need corrective
fetches."""

import numpy as np
import pytest
import torch

import oracle as O
from lookahead_sparse_kv_b200 import workloads as W


def _bf16_round(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("seed", range(4))
def test_overlap_brute_force(seed):
    """Distinct ids of b found anywhere in a, by a double loop; -1 ignored,
    duplicates counted once."""
    r = np.random.default_rng(seed)
    a = r.integers(-1, 20, size=(3, 2, 9)).astype(np.int32)
    b = r.integers(-1, 20, size=(3, 2, 7)).astype(np.int32)
    got = O.block_overlap(a, b)
    for i in range(3):
        for h in range(2):
            seen, n = [], 0
            for x in b[i, h]:
                if x < 0 or x in seen:
                    continue
                seen.append(x)
                if any(y == x for y in a[i, h]):
                    n += 1
            assert got[i, h] == n
    assert (O.block_overlap(a, a) == [[len({x for x in a[i, h] if x >= 0}) for h in range(2)]
                                      for i in range(3)]).all()
    np.testing.assert_array_equal(O.block_overlap(a, b), O.block_overlap(b, a))


def test_scores_rows_are_a_max_over_single_rows():
    """Scoring a set of rows takes the max of the single-row scores."""
    r = np.random.default_rng(3)
    B, Qn, Hq, H, N, P, D = 2, 4, 4, 2, 7, 16, 8
    keys = _bf16_round(r.standard_normal((B, H, N, P, D)))
    q = _bf16_round(r.standard_normal((B, Qn, Hq, D)))
    ctx = np.array([N * P, 3 * P + 5])
    kmin, kmax = O.block_summaries(keys, ctx)
    single = [O.lookahead_scores(q, kmin, kmax, ctx, P, rows=[j]) for j in range(Qn)]
    np.testing.assert_array_equal(O.lookahead_scores(q, kmin, kmax, ctx, P, rows=[1, 2]),
                                  np.maximum(single[1], single[2]))
    np.testing.assert_array_equal(O.lookahead_scores(q, kmin, kmax, ctx, P),
                                  np.maximum(np.maximum(single[1], single[2]), single[3]))


def test_scores_row_zero_on_one_token_blocks_is_the_dot_product():
    """With one token per block the bound is attained: the verification-row
    score is max over the G heads of q0 . k."""
    r = np.random.default_rng(4)
    B, Qn, Hq, H, N, D = 1, 3, 4, 2, 6, 8
    keys = _bf16_round(r.standard_normal((B, H, N, 1, D)))
    q = _bf16_round(r.standard_normal((B, Qn, Hq, D)))
    ctx = np.array([N])
    kmin, kmax = O.block_summaries(keys, ctx)
    s = O.lookahead_scores(q, kmin, kmax, ctx, 1, rows=[0])
    for h in range(H):
        for n in range(N):
            best = max(float(q[0, 0, h * 2 + g] @ keys[0, h, n, 0]) for g in range(2))
            assert s[0, h, n] == np.float32(best)


def _small_decode(corrective, fetch_cap, seed=5, steps=4):
    r = np.random.default_rng(seed)
    B, Qn, Hq, H, N, P, D, K = 2, 3, 4, 2, 24, 16, 16, 6
    keys = _bf16_round(r.standard_normal((B, H, N, P, D)))
    vals = _bf16_round(r.standard_normal((B, H, N, P, D)))
    ctx = np.array([N * P - 7, 17 * P])
    kmin, kmax = O.block_summaries(keys, ctx)
    qp = _bf16_round(r.standard_normal((B, Qn, Hq, D)))
    qsteps = [_bf16_round(r.standard_normal((B, Qn, Hq, D))) for _ in range(steps)]
    recs, st, lu = O.decode_layer_steps(keys, vals, kmin, kmax, ctx, qp, qsteps, budget_blocks=K,
                                        fetch_cap=fetch_cap, scale=0.25, corrective=corrective)
    return recs, (keys, vals, kmin, kmax, ctx, qp, qsteps, K)


def test_corrective_fetch_makes_the_exact_set_resident():
    """Before each attention the exact set is resident; the uncapped plan
    fetches exactly the blocks of E_t that were not resident."""
    recs, (keys, vals, kmin, kmax, ctx, qp, qsteps, K) = _small_decode(True, fetch_cap=1)
    for t, rec in enumerate(recs):
        c = rec["corrective"]
        exact = c["exact"]
        n_exact = (exact >= 0).sum(axis=2)
        # recomputed from its definition: top-K under the verification row alone
        ref, _ = O.select_topk(O.lookahead_scores(qsteps[t], kmin, kmax, ctx, 16, rows=[0]), ctx, K, 16)
        np.testing.assert_array_equal(exact, ref)
        assert (O.block_overlap(rec["slot_table_attn"], exact) == n_exact).all()
        np.testing.assert_array_equal(c["covered"] + c["plan"]["n_fetch"], n_exact)
        assert (c["agree_lookahead"] <= n_exact).all()
        if t == 0:
            assert c["agree_prev"] is None
        else:
            np.testing.assert_array_equal(c["agree_prev"],
                                          O.block_overlap(recs[t - 1]["corrective"]["exact"], exact))
            np.testing.assert_array_equal(c["agree_lookahead"], O.block_overlap(recs[t - 1]["sel"], exact))


def test_corrective_attention_sees_a_superset_of_the_capped_one():
    """With the corrective fetch the attention's resident set always contains
    the exact set, which the capped lookahead alone does not guarantee."""
    plain, _ = _small_decode(False, fetch_cap=1)
    corr, _ = _small_decode(True, fetch_cap=1)
    missed = 0
    for rp, rc in zip(plain, corr):
        exact = rc["corrective"]["exact"]
        n_exact = (exact >= 0).sum(axis=2)
        missed += int((n_exact - O.block_overlap(rp["slot_table_attn"], exact)).sum())
        assert (O.block_overlap(rc["slot_table_attn"], exact) == n_exact).all()
    assert missed > 0          # the case is not vacuous: the cap of 1 leaves misses


def test_lead_drafts_carry_future_means():
    """With zero noise, draft row j of step t equals the verification row of
    step t+j (the query mean j steps ahead), and the drift moves the mean."""
    w = W.WORKLOADS["tiny"].with_(draft_lead=True, ar_rho=0.9, query_noise=0.0)
    qs = W.QueryStream(w)
    steps = [qs.next() for _ in range(8)]
    Qn = w.n_queries
    for t in range(8 - Qn + 1):
        for j in range(1, Qn):
            assert torch.equal(steps[t][:, j], steps[t + j][:, 0])
    assert not torch.equal(steps[0][:, 0], steps[1][:, 0])


def test_default_stream_is_unchanged_by_the_lead_option():
    """Rows of a step share one mean without draft_lead (zero noise: equal rows)."""
    w = W.WORKLOADS["tiny"].with_(ar_rho=0.9, query_noise=0.0)
    q = W.QueryStream(w).next()
    for j in range(1, w.n_queries):
        assert torch.equal(q[:, j], q[:, 0])
