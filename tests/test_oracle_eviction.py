"""Pins for the score-based victim order of the planner (the alternative to
LRU in the eviction ablation; OasisKV Table 2 names LRU).  CPU only."""

import numpy as np
import pytest

import oracle as O


def _state():
    # one (sequence, head), K = 4 slots: blocks 10, 11, 12 resident, slot 3 free
    st = np.array([[[10, 11, 12, -1]]], dtype=np.int32)
    lu = np.array([[[3, 1, 2, -1]]], dtype=np.int32)
    sel = np.array([[[20, 21, 11, -1]]], dtype=np.int32)   # 11 resident, 20 and 21 missing
    scores = np.zeros((1, 1, 32), dtype=np.float32)
    scores[0, 0, 10], scores[0, 0, 12] = -5.0, 7.0
    return st, lu, sel, scores


def test_hand_worked_lru_vs_score_victims():
    """Worked by hand: the free slot 3 goes first; the second victim is the
    least recently used stale slot (slot 2, last used at 2) under LRU, but the
    lowest-scored stale block (block 10 in slot 0, score -5) under R17."""
    st, lu, sel, scores = _state()
    lru = O.plan_fetch(sel, st, lu, 5, 2)
    assert lru["fetch_slot"][0, 0].tolist() == [3, 2]
    assert lru["slot_table"][0, 0].tolist() == [10, 11, 21, 20]
    sc = O.plan_fetch(sel, st, lu, 5, 2, scores=scores)
    assert sc["fetch_slot"][0, 0].tolist() == [3, 0]
    assert sc["slot_table"][0, 0].tolist() == [21, 11, 12, 20]
    for p in (lru, sc):
        assert p["last_used"][0, 0, 1] == 5          # the selected resident block is stamped
        assert p["n_fetch"][0, 0] == 2


def test_score_ties_go_to_the_lower_block_and_signed_zeros_tie():
    st = np.array([[[9, 4, 7, -1]]], dtype=np.int32)
    lu = np.array([[[0, 0, 0, -1]]], dtype=np.int32)
    sel = np.array([[[30, 31, 32, -1]]], dtype=np.int32)
    scores = np.zeros((1, 1, 40), dtype=np.float32)
    scores[0, 0, 9], scores[0, 0, 4], scores[0, 0, 7] = -0.0, 0.0, 1.0
    p = O.plan_fetch(sel, st, lu, 1, 3, scores=scores)
    # free slot 3, then blocks 4 (slot 1) and 9 (slot 0): equal scores, lower id first
    assert p["fetch_slot"][0, 0].tolist() == [3, 1, 0]


@pytest.mark.parametrize("seed", range(6))
def test_score_victims_keep_the_planner_invariants(seed):
    """Brute-force check of the victim order on random states, and the
    invariants shared with LRU: selected blocks stay, free slots first."""
    r = np.random.default_rng(seed)
    B, H, K, N, C = 2, 2, 12, 40, 5
    st = np.full((B, H, K), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            n_occ = r.integers(0, K + 1)
            st[b, h, r.permutation(K)[:n_occ]] = r.permutation(N)[:n_occ]
    lu = r.integers(-1, 6, size=(B, H, K)).astype(np.int32)
    sel = np.stack([np.stack([r.permutation(N)[:K] for _ in range(H)]) for _ in range(B)]).astype(np.int32)
    scores = r.integers(-3, 3, size=(B, H, N)).astype(np.float32)     # many ties
    p = O.plan_fetch(sel, st, lu, 9, C, scores=scores)
    for b in range(B):
        for h in range(H):
            chosen = set(sel[b, h].tolist())
            free = [s for s in range(K) if st[b, h, s] < 0]
            stale = [s for s in range(K) if st[b, h, s] >= 0 and st[b, h, s] not in chosen]
            n = int(p["n_fetch"][b, h])
            victims = p["fetch_slot"][b, h, :n].tolist()
            # brute force: each victim beats every stale slot left in place
            expect = free[:n]
            rest = n - len(expect)
            if rest > 0:
                order = sorted(stale, key=lambda s: (scores[b, h, st[b, h, s]], st[b, h, s]))
                expect += order[:rest]
            assert victims == expect
            for s in range(K):
                if st[b, h, s] in chosen:
                    assert p["slot_table"][b, h, s] == st[b, h, s]


def test_residency_loss_frees_slots_and_forces_refetch():
    """R19: a lost slot is free at the next plan; its block, if selected
    again, is a miss and lands in a free slot (free slots come first)."""
    st = np.array([[[10, 11, 12, 13]]], dtype=np.int32)
    lu = np.array([[[4, 4, 4, 4]]], dtype=np.int32)
    mask = np.array([[[False, True, False, True]]])
    st2 = O.evict_slots(st, mask)
    assert st2[0, 0].tolist() == [10, -1, 12, -1]
    assert st[0, 0].tolist() == [10, 11, 12, 13]                 # input untouched
    sel = np.array([[[11, 10, 12, 13]]], dtype=np.int32)
    p = O.plan_fetch(sel, st2, lu, 5, 4)
    assert p["n_fetch"][0, 0] == 2
    assert p["fetch_block"][0, 0, :2].tolist() == [11, 13]       # rank order
    assert p["fetch_slot"][0, 0, :2].tolist() == [1, 3]          # the freed slots, ascending


def test_decode_with_residency_loss_refetches_what_was_lost():
    """Over a few decode steps with a loss mask, the fetch count is at least the
    number of lost blocks the next selection wants back (up to the cap)."""
    r = np.random.default_rng(9)
    B, Qn, Hq, H, N, P, D, K = 1, 3, 4, 2, 20, 16, 8, 6
    keys = r.standard_normal((B, H, N, P, D)).astype(np.float32).astype(np.float64)
    vals = r.standard_normal((B, H, N, P, D))
    ctx = np.array([N * P])
    kmin, kmax = O.block_summaries(keys, ctx)
    qp = r.standard_normal((B, Qn, Hq, D))
    qsteps = [qp + 0.01 * r.standard_normal((B, Qn, Hq, D)) for _ in range(4)]   # nearly the same selection
    masks = [r.random((B, H, K)) < 0.5 for _ in range(4)]
    recs, _, _ = O.decode_layer_steps(keys, vals, kmin, kmax, ctx, qp, qsteps, budget_blocks=K, fetch_cap=K,
                                      scale=0.3, evict_masks=masks)
    for t, rec in enumerate(recs):
        before = O.evict_slots(rec["slot_table_attn"], masks[t])
        lost = set(rec["slot_table_attn"][0, 0][masks[t][0, 0]].tolist()) - {-1}
        wanted_back = lost & set(rec["sel"][0, 0].tolist())
        assert rec["plan"]["n_fetch"][0, 0] >= len(wanted_back)
        assert set(rec["plan"]["fetch_block"][0, 0].tolist()) >= wanted_back
        assert (before[0, 0][masks[t][0, 0]] == -1).all()
