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
