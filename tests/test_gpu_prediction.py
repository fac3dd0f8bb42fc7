"""Exact top-K set, prediction-agreement counts and the corrective fetch on the
GPU against the oracle (OasisKV Figures 4 and 6; corrective fetches after
prediction misses).  Selections follow the 1e-5 tie rule, counts and plans are
bit-exact on the GPU's own selections, attention within abs 2e-3 / rel 1e-2."""

import math

import numpy as np
import pytest
import torch

import lookahead_sparse_kv_b200 as lsk
import oracle as O
from lookahead_sparse_kv_b200 import workloads as W
from lookahead_sparse_kv_b200.pipeline import DecodePipeline, LayerState
from tests.gpu_util import (assert_attention_close, assert_selection_matches, f64, kv_split, np_i32,
                            random_kv)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from lookahead_sparse_kv_b200 import build
    build.build()
    lsk.lib()
    yield
    assert lsk.read_device_error(clear=True) == 0


@pytest.mark.parametrize("B,Hq,Hkv,Qn,N,K,rows", [
    (2, 8, 2, 5, 300, 32, (0, 1)),        # verification row alone
    (2, 8, 2, 5, 300, 32, (2, 2)),        # a window of drafts
    (3, 32, 8, 5, 1000, 64, (0, 5)),      # every row
    (1, 64, 8, 8, 700, 128, (0, 1)),      # G = 8
    (2, 4, 4, 1, 129, 16, (0, 1)),        # no drafts
])
def test_score_select_rows_matches_oracle(B, Hq, Hkv, Qn, N, K, rows):
    d = lsk.make_dims(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, max_blocks=N, budget_blocks=K,
                      n_queries=Qn, fetch_cap=min(8, K))
    g = torch.Generator()
    g.manual_seed(1000 + N + rows[0])
    kv = random_kv(B, Hkv, N, g)
    keys = f64(kv)[:, :, :, 0]
    ctx = torch.tensor([N * 16 - 5 * i for i in range(B)], dtype=torch.int32)
    q = torch.randn(B, Qn, Hq, 128, generator=g).to(torch.bfloat16)
    kmin = torch.empty((B, Hkv, N, 128), dtype=torch.bfloat16, device=DEV)
    kmax = torch.empty_like(kmin)
    ws = torch.zeros(lsk.workspace_bytes(d), dtype=torch.uint8, device=DEV)
    sel = torch.full((B, Hkv, K), -7, dtype=torch.int32, device=DEV)
    ctx_d = ctx.to(DEV)
    lsk.build_summaries(d, kv.to(DEV), ctx_d, kmin, kmax)
    lsk.score_select_rows(d, q.to(DEV), rows[0], rows[1], kmin, kmax, ctx_d, sel, None, ws)
    torch.cuda.synchronize()
    omin, omax = O.block_summaries(keys, ctx.numpy())
    sc = O.lookahead_scores(f64(q), omin, omax, ctx.numpy(), 16, rows=list(range(rows[0], rows[0] + rows[1])))
    ref, _ = O.select_topk(sc, ctx.numpy(), K, 16)
    assert_selection_matches(np_i32(sel), ref, sc, ctx.numpy(), K)


def test_score_select_rows_rejects_rows_outside_the_step():
    d = lsk.make_dims(batch=1, n_q_heads=8, n_kv_heads=2, max_blocks=64, budget_blocks=16,
                      n_queries=5, fetch_cap=4)
    q = torch.zeros((1, 5, 8, 128), dtype=torch.bfloat16, device=DEV)
    summ = torch.zeros((1, 2, 64, 128), dtype=torch.bfloat16, device=DEV)
    ctx = torch.full((1,), 64 * 16, dtype=torch.int32, device=DEV)
    sel = torch.zeros((1, 2, 16), dtype=torch.int32, device=DEV)
    ws = torch.zeros(lsk.workspace_bytes(d), dtype=torch.uint8, device=DEV)
    for rb, rc in [(-1, 1), (0, 0), (4, 2), (5, 1)]:
        with pytest.raises(lsk.OasisError) as e:
            lsk.score_select_rows(d, q, rb, rc, summ, summ, ctx, sel, None, ws)
        assert e.value.code == lsk.EINVAL and "query rows" in str(e.value)


@pytest.mark.parametrize("B,Hkv,N,K,seed", [(2, 3, 50, 20, 0), (4, 8, 2048, 128, 1), (1, 2, 32768, 1024, 2),
                                            (1, 1, 5, 1, 3)])
def test_block_overlap_bit_exact(B, Hkv, N, K, seed):
    d = lsk.make_dims(batch=B, n_q_heads=Hkv, n_kv_heads=Hkv, max_blocks=N, budget_blocks=K,
                      n_queries=1, fetch_cap=0)
    r = np.random.default_rng(seed)
    a = r.integers(-1, N, size=(B, Hkv, K)).astype(np.int32)
    b = r.integers(-1, N, size=(B, Hkv, K)).astype(np.int32)
    b[0, 0] = -1                                    # an empty list
    if K > 4:
        b[-1, -1, : K // 2] = a[-1, -1, : K // 2]   # a large shared part
        b[-1, -1, 1] = b[-1, -1, 0]                 # a repeated id
    cnt = torch.full((B, Hkv), -9, dtype=torch.int32, device=DEV)
    lsk.block_overlap(d, torch.from_numpy(a).to(DEV), torch.from_numpy(b).to(DEV), cnt)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(np_i32(cnt), O.block_overlap(a, b))
    assert np_i32(cnt)[0, 0] == 0


def test_block_overlap_skips_and_flags_bad_ids():
    d = lsk.make_dims(batch=1, n_q_heads=2, n_kv_heads=2, max_blocks=40, budget_blocks=4,
                      n_queries=1, fetch_cap=0)
    a = torch.tensor([[[1, 2, 3, 40], [5, -3, 6, 7]]], dtype=torch.int32, device=DEV)
    b = torch.tensor([[[3, 40, 1, -1], [7, 7, 99, 5]]], dtype=torch.int32, device=DEV)
    cnt = torch.zeros((1, 2), dtype=torch.int32, device=DEV)
    lsk.read_device_error(clear=True)
    lsk.block_overlap(d, a, b, cnt)
    torch.cuda.synchronize()
    assert np_i32(cnt).tolist() == [[2, 2]]
    assert lsk.read_device_error(clear=True) & lsk.DEVERR_ID_RANGE


@pytest.mark.parametrize("mode", ["measure", "correct"])
def test_exact_set_pipeline_step_by_step(mode):
    """The stream pipeline with the exact-set stage on a small leading-draft
    workload, every step checked: exact set, the four counts, the corrective
    plan, attention over the corrected residency, the lookahead plan."""
    w = W.WORKLOADS["llama8b_32k_lead"].with_(batch=2, n_q_heads=8, n_kv_heads=2, context=8192,
                                               max_blocks=512, budget_blocks=32, fetch_cap=2)
    d = lsk.dims_for(w)
    K, C = w.budget_blocks, w.fetch_cap
    host = W.make_host_kv(w).pin_memory()
    host_bits = W.bf16_bits(host)
    keys, vals = kv_split(host)
    ctx = W.initial_ctx_len(w)
    cnp = ctx.numpy()
    L = LayerState(d, host, DEV)
    scale = 1 / math.sqrt(128)
    pipe = DecodePipeline(d, [L], ctx.to(DEV), scale, DEV, exact=mode, steps_cap=8)
    pipe.build_summaries()
    kmin, kmax = O.block_summaries(keys, cnp)
    qs = W.QueryStream(w)
    pipe.prime([qs.next().to(DEV)])
    pipe.wait_all()
    torch.cuda.synchronize()
    st, lu = np_i32(L.slot_table), np_i32(L.last_used)
    sel_prev, exact_prev = np_i32(L.sel), None
    fetched_corrective = 0
    for t in range(1, 9):
        q = qs.next()
        pipe.step(t, [q.to(DEV)])
        pipe.wait_all()
        torch.cuda.synchronize()
        counts = pipe.prediction_counts()[0, :, (t - 1) % 8]
        exact = np_i32(L.exact[t % 2])
        sc = O.lookahead_scores(f64(q), kmin, kmax, cnp, 16, rows=[0])
        ref_exact, _ = O.select_topk(sc, cnp, K, 16)
        assert_selection_matches(exact, ref_exact, sc, cnp, K)
        np.testing.assert_array_equal(counts[0].numpy(), O.block_overlap(sel_prev, exact))
        if t > 1:
            np.testing.assert_array_equal(counts[1].numpy(), O.block_overlap(exact_prev, exact))
        np.testing.assert_array_equal(counts[2].numpy(), O.block_overlap(st, exact))
        if mode == "correct":
            plan = O.plan_fetch(exact, st, lu, t, K)
            np.testing.assert_array_equal(counts[3].numpy(), plan["n_fetch"])
            fetched_corrective += int(plan["n_fetch"].sum())
            st, lu = plan["slot_table"], plan["last_used"]
            assert (O.block_overlap(st, exact) == (exact >= 0).sum(axis=2)).all()
        # attention over the residency it ran on
        pk = np.zeros((w.batch, w.n_kv_heads, K, 16, 128))
        pv = np.zeros_like(pk)
        for b in range(w.batch):
            for h in range(w.n_kv_heads):
                for s in range(K):
                    if st[b, h, s] >= 0:
                        pk[b, h, s], pv[b, h, s] = keys[b, h, st[b, h, s]], vals[b, h, st[b, h, s]]
        o_ref, lse_ref = O.sparse_attention(f64(q), pk, pv, st, cnp, scale)
        assert_attention_close(L.out, L.lse, o_ref, lse_ref)
        # lookahead selection and capped plan of this step
        sc2 = O.lookahead_scores(f64(q), kmin, kmax, cnp, 16)
        ref_sel, _ = O.select_topk(sc2, cnp, K, 16)
        sel = np_i32(L.sel)
        assert_selection_matches(sel, ref_sel, sc2, cnp, K)
        plan = O.plan_fetch(sel, st, lu, t, C)
        np.testing.assert_array_equal(np_i32(L.slot_table), plan["slot_table"])
        np.testing.assert_array_equal(np_i32(L.last_used), plan["last_used"])
        st, lu = plan["slot_table"], plan["last_used"]
        pb = W.bf16_bits(L.pool)
        for b in range(w.batch):
            for h in range(w.n_kv_heads):
                for s in np.nonzero(st[b, h] >= 0)[0]:
                    np.testing.assert_array_equal(pb[b, h, s], host_bits[b, h, st[b, h, s]])
        sel_prev, exact_prev = sel, exact
    if mode == "correct":
        assert fetched_corrective > 0        # the cap of 2 leaves misses to correct
