"""A decode step captured as one CUDA graph (device-resident step counter,
a7 with the f2 graph capture) gives bit-identical results to the eager
stream pipeline, step after step, over several layers, with a residency-loss
mask per layer and step."""

import math

import pytest
import torch

import lookahead_sparse_kv_b200 as lsk
from lookahead_sparse_kv_b200 import workloads as W
from lookahead_sparse_kv_b200.pipeline import DecodePipeline, LayerState

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from lookahead_sparse_kv_b200 import build
    build.build()
    lsk.lib()
    yield
    assert lsk.read_device_error(clear=True) == 0


def _setup(w, hosts, **kw):
    d = lsk.dims_for(w)
    layers = [LayerState(d, h, DEV) for h in hosts]
    pipe = DecodePipeline(d, layers, W.initial_ctx_len(w).to(DEV), 1 / math.sqrt(128), DEV, **kw)
    with torch.cuda.stream(pipe.main):
        pipe.build_summaries()
    return pipe, layers


def _state(layers):
    return [t.clone() for L in layers for t in (L.out, L.lse, L.slot_table, L.last_used, L.pool)]


@pytest.mark.parametrize("victims", ["lru", "score"])
def test_graph_replay_matches_eager(victims):
    w = W.WORKLOADS["llama8b_32k"].with_(batch=2, n_q_heads=8, n_kv_heads=2, context=8192, max_blocks=512,
                                          budget_blocks=32, fetch_cap=3, layers=3, evict_prob=0.1)
    hosts = [W.make_host_kv(w, l).pin_memory() for l in range(w.layers)]
    streams = [W.QueryStream(w, l) for l in range(w.layers)]
    qs = [[s.next().to(DEV) for _ in range(12)] for s in streams]           # [layer][step]
    masks = [[W.eviction_mask(w, l, t, DEV).to(torch.uint8) for l in range(w.layers)] for t in range(12)]
    steps = range(1, 12)

    ref, ref_layers = _setup(w, hosts, victims=victims)                      # by-value step numbers
    ref.prime([q[0] for q in qs])
    want = []
    for t in steps:
        ref.step(t, [q[t] for q in qs], evict=masks[t])
        ref.wait_all()
        torch.cuda.synchronize()
        want.append(_state(ref_layers))

    dev, dev_layers = _setup(w, hosts, victims=victims, device_step=True)    # device counter, eager
    gr, gr_layers = _setup(w, hosts, victims=victims, device_step=True)      # device counter, graph
    q_static = [torch.empty_like(q[0]) for q in qs]
    m_static = [torch.empty_like(m) for m in masks[0]]
    for p in (dev, gr):
        with torch.cuda.stream(p.main):
            p.prime([q[0] for q in qs])
    for t in steps:
        with torch.cuda.stream(dev.main):
            dev.step(t, [q[t] for q in qs], evict=masks[t])
            dev.wait_all()
        if t <= 2:
            with torch.cuda.stream(gr.main):
                gr.step(t, [q[t] for q in qs], evict=masks[t])
                gr.wait_all()
        else:
            if gr.graph is None:
                gr.capture(q_static, evict_static=m_static)
            with torch.cuda.stream(gr.main):
                for qd, q in zip(q_static, qs):
                    qd.copy_(q[t])
                for md, m in zip(m_static, masks[t]):
                    md.copy_(m)
            gr.replay()
        torch.cuda.synchronize()
        for a, b in zip(want[t - 1], _state(dev_layers)):
            assert torch.equal(a, b), f"device-step eager differs at step {t}"
        for a, b in zip(want[t - 1], _state(gr_layers)):
            assert torch.equal(a, b), f"graph replay differs at step {t}"
    assert int(gr.step_dev[0].item()) == 11


@pytest.mark.parametrize("victims", ["lru", "score"])
def test_graph_replay_matches_oracle(victims):
    """The replayed decode steps against the CPU oracle, not only against the
    eager GPU pipeline: per step and layer, the attention over the working
    set staged by the previous step, the selection (tie rule), the plan after
    that step's residency loss (slot table, recency, fetch lists bit-exact;
    score-ordered victims use the GPU's own fp32 scores) and the bytes of
    every occupied pool slot.  The first two steps run eagerly with the
    device step counter, the rest as replays of one captured graph."""
    import numpy as np

    import oracle as O
    from tests.gpu_util import assert_attention_close, assert_selection_matches, f64, kv_split, np_i32

    w = W.WORKLOADS["llama8b_32k"].with_(batch=2, n_q_heads=8, n_kv_heads=2, context=8192 - 5, max_blocks=512,
                                          budget_blocks=32, fetch_cap=3, layers=2, evict_prob=0.1)
    K, C, scale = w.budget_blocks, w.fetch_cap, 1 / math.sqrt(128)
    hosts = [W.make_host_kv(w, l).pin_memory() for l in range(w.layers)]
    streams = [W.QueryStream(w, l) for l in range(w.layers)]
    qs = [[s.next() for _ in range(9)] for s in streams]                    # [layer][step], CPU
    masks = [[W.eviction_mask(w, l, t) for l in range(w.layers)] for t in range(9)]
    ctx = W.initial_ctx_len(w).numpy()
    ref = []
    for l in range(w.layers):
        keys, vals = kv_split(hosts[l])
        kmin, kmax = O.block_summaries(keys, ctx)
        ref.append({"keys": keys, "vals": vals, "kmin": kmin, "kmax": kmax, "bits": W.bf16_bits(hosts[l]),
                    "st": np.full((w.batch, w.n_kv_heads, K), -1, np.int32),
                    "lu": np.full((w.batch, w.n_kv_heads, K), -1, np.int32)})

    gr, layers = _setup(w, hosts, victims=victims, device_step=True)
    q_static = [torch.empty_like(q[0], device=DEV) for q in qs]
    m_static = [torch.empty((w.batch, w.n_kv_heads, K), dtype=torch.uint8, device=DEV) for _ in range(w.layers)]

    def check_select_plan(l, q, t, st_before):
        r, L = ref[l], layers[l]
        sc = O.lookahead_scores(f64(q), r["kmin"], r["kmax"], ctx, 16)
        ref_sel, _ = O.select_topk(sc, ctx, K, 16)
        sel = np_i32(L.sel)
        assert_selection_matches(sel, ref_sel, sc, ctx, K)
        gsc = L.scores.cpu().numpy() if victims == "score" else None
        plan = O.plan_fetch(sel, st_before, r["lu"], t, C, scores=gsc)
        for key, got in (("slot_table", L.slot_table), ("last_used", L.last_used), ("fetch_slot", L.fetch_slot),
                         ("fetch_block", L.fetch_block), ("n_fetch", L.n_fetch)):
            np.testing.assert_array_equal(np_i32(got), plan[key], err_msg=f"{key}, layer {l}, step {t}")
        r["st"], r["lu"] = plan["slot_table"], plan["last_used"]
        pb = W.bf16_bits(L.pool)
        for b in range(w.batch):
            for h in range(w.n_kv_heads):
                for s in np.nonzero(r["st"][b, h] >= 0)[0]:
                    np.testing.assert_array_equal(pb[b, h, s], r["bits"][b, h, r["st"][b, h, s]])

    with torch.cuda.stream(gr.main):
        gr.prime([q[0].to(DEV) for q in qs])
        gr.wait_all()
    torch.cuda.synchronize()
    for l in range(w.layers):
        check_select_plan(l, qs[l][0], 0, ref[l]["st"])
    replays = 0
    for t in range(1, 9):
        st_attn = [r["st"].copy() for r in ref]
        if t <= 2:
            with torch.cuda.stream(gr.main):
                gr.step(t, [q[t].to(DEV) for q in qs], evict=[m.to(torch.uint8).to(DEV) for m in masks[t]])
                gr.wait_all()
        else:
            if gr.graph is None:
                gr.capture(q_static, evict_static=m_static)
            with torch.cuda.stream(gr.main):
                for qd, q in zip(q_static, qs):
                    qd.copy_(q[t])
                for md, m in zip(m_static, masks[t]):
                    md.copy_(m.to(torch.uint8))
            gr.replay()
            replays += 1
        torch.cuda.synchronize()
        for l, L in enumerate(layers):
            r = ref[l]
            pk = np.zeros((w.batch, w.n_kv_heads, K, 16, 128))
            pv = np.zeros_like(pk)
            for b in range(w.batch):
                for h in range(w.n_kv_heads):
                    for s in np.nonzero(st_attn[l][b, h] >= 0)[0]:
                        pk[b, h, s] = r["keys"][b, h, st_attn[l][b, h, s]]
                        pv[b, h, s] = r["vals"][b, h, st_attn[l][b, h, s]]
            o_ref, lse_ref = O.sparse_attention(f64(qs[l][t]), pk, pv, st_attn[l], ctx, scale)
            assert_attention_close(L.out, L.lse, o_ref, lse_ref)
            check_select_plan(l, qs[l][t], t, O.evict_slots(st_attn[l], masks[t][l].numpy()))
    assert replays == 6 and int(gr.step_dev[0].item()) == 8
