"""Score-ordered victims (the eviction ablation's alternative to OasisKV
Table 2's LRU) on the GPU against the oracle: the planner bit-exact on random
states, and the stream pipeline step by step with this policy."""

import math

import numpy as np
import pytest
import torch

import lookahead_sparse_kv_b200 as lsk
import oracle as O
from lookahead_sparse_kv_b200 import workloads as W
from lookahead_sparse_kv_b200.pipeline import DecodePipeline, LayerState
from tests.gpu_util import SCORE_REL, assert_selection_matches, f64, kv_split, np_i32

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from lookahead_sparse_kv_b200 import build
    build.build()
    lsk.lib()
    yield
    assert lsk.read_device_error(clear=True) == 0


@pytest.mark.parametrize("B,H,K,N,C,seed", [(3, 4, 16, 64, 5, 0), (2, 8, 128, 2048, 16, 1),
                                            (1, 2, 1024, 4096, 1024, 2), (2, 2, 7, 9, 7, 3)])
def test_plan_fetch_scored_bit_exact(B, H, K, N, C, seed):
    r = np.random.default_rng(seed)
    st = np.full((B, H, K), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            n_occ = int(r.integers(0, K + 1))
            st[b, h, r.permutation(K)[:n_occ]] = r.permutation(N)[:n_occ]
    lu = r.integers(-1, 50, size=(B, H, K)).astype(np.int32)
    sel = np.full((B, H, K), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            n_sel = int(r.integers(0, K + 1))
            sel[b, h, :n_sel] = r.permutation(N)[:n_sel]
    scores = r.integers(-4, 4, size=(B, H, N)).astype(np.float32)        # ties
    scores[r.random((B, H, N)) < 0.1] = -0.0                              # signed zeros tie with +0.0
    d = lsk.make_dims(batch=B, n_q_heads=H, n_kv_heads=H, max_blocks=N, budget_blocks=K,
                      n_queries=1, fetch_cap=C)
    t = {k: torch.from_numpy(v).to(DEV) for k, v in (("st", st), ("lu", lu), ("sel", sel), ("sc", scores))}
    fs = torch.full((B, H, C), -9, dtype=torch.int32, device=DEV)
    fb = torch.full_like(fs, -9)
    nf = torch.full((B, H), -9, dtype=torch.int32, device=DEV)
    lsk.plan_fetch_scored(d, t["sel"], t["sc"], t["st"], t["lu"], 42, fs, fb, nf)
    torch.cuda.synchronize()
    p = O.plan_fetch(sel, st, lu, 42, C, scores=scores)
    np.testing.assert_array_equal(np_i32(t["st"]), p["slot_table"])
    np.testing.assert_array_equal(np_i32(t["lu"]), p["last_used"])
    np.testing.assert_array_equal(np_i32(fs), p["fetch_slot"])
    np.testing.assert_array_equal(np_i32(fb), p["fetch_block"])
    np.testing.assert_array_equal(np_i32(nf), p["n_fetch"])


def test_pipeline_with_score_victims_step_by_step():
    w = W.WORKLOADS["llama8b_32k"].with_(batch=2, n_q_heads=8, n_kv_heads=2, context=8192,
                                          max_blocks=512, budget_blocks=32, fetch_cap=3)
    d = lsk.dims_for(w)
    K, C = w.budget_blocks, w.fetch_cap
    host = W.make_host_kv(w).pin_memory()
    host_bits = W.bf16_bits(host)
    keys, _ = kv_split(host)
    ctx = W.initial_ctx_len(w)
    cnp = ctx.numpy()
    L = LayerState(d, host, DEV)
    pipe = DecodePipeline(d, [L], ctx.to(DEV), 1 / math.sqrt(128), DEV, victims="score")
    pipe.build_summaries()
    kmin, kmax = O.block_summaries(keys, cnp)
    qs = W.QueryStream(w)
    st = np.full((w.batch, w.n_kv_heads, K), -1, np.int32)
    lu = st.copy()
    evicted_differently = 0
    for t in range(0, 20):
        q = qs.next()
        if t == 0:
            pipe.prime([q.to(DEV)])
        else:
            pipe.step(t, [q.to(DEV)])
        pipe.wait_all()
        torch.cuda.synchronize()
        sc = O.lookahead_scores(f64(q), kmin, kmax, cnp, 16)
        gsc = L.scores.cpu().numpy()
        nv = int(O.n_valid_blocks(cnp, 16).min())
        np.testing.assert_allclose(gsc[:, :, :nv], sc[:, :, :nv], rtol=SCORE_REL, atol=0)
        ref_sel, _ = O.select_topk(sc, cnp, K, 16)
        sel = np_i32(L.sel)
        assert_selection_matches(sel, ref_sel, sc, cnp, K)
        plan = O.plan_fetch(sel, st, lu, t, C, scores=gsc)
        lru = O.plan_fetch(sel, st, lu, t, C)
        evicted_differently += int((plan["slot_table"] != lru["slot_table"]).sum())
        np.testing.assert_array_equal(np_i32(L.slot_table), plan["slot_table"])
        np.testing.assert_array_equal(np_i32(L.last_used), plan["last_used"])
        st, lu = plan["slot_table"], plan["last_used"]
        pb = W.bf16_bits(L.pool)
        for b in range(w.batch):
            for h in range(w.n_kv_heads):
                for s in np.nonzero(st[b, h] >= 0)[0]:
                    np.testing.assert_array_equal(pb[b, h, s], host_bits[b, h, st[b, h, s]])
    assert evicted_differently > 0        # the two policies do diverge on this run
