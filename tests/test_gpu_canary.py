"""Guard bands around every buffer the library writes: each device and pinned
host buffer is carved out of a larger allocation whose 4 KiB on either side
hold a fixed byte pattern, every call that writes memory runs on ragged sizes
(two sequences of different lengths, a partial last block), and the pattern
must be intact afterwards.  A kernel that writes past either end of a buffer
fails here even when its results inside the buffer are right."""

import math

import pytest
import torch

import lookahead_sparse_kv_b200 as lsk
from lookahead_sparse_kv_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
GUARD_BYTES = 4096
CANARY = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from lookahead_sparse_kv_b200 import build
    build.build()
    lsk.lib()
    yield


class Guarded:
    """A buffer of `shape` inside an allocation with GUARD_BYTES of canary on each side."""

    def __init__(self, shape, dtype, device=DEV, init=None):
        el = torch.empty((), dtype=dtype).element_size()
        self.n, self.g = math.prod(shape), GUARD_BYTES // el
        raw = torch.empty(self.n + 2 * self.g, dtype=dtype)
        if device == "pinned":
            raw = raw.pin_memory()
        else:
            raw = raw.to(device)
        raw.view(torch.uint8).fill_(CANARY)
        self.raw = raw
        self.t = raw[self.g:self.g + self.n].view(shape)
        if init is not None:
            self.t.copy_(init)

    def intact(self) -> bool:
        b = self.raw.view(torch.uint8)
        el = self.raw.element_size()
        head, tail = b[: self.g * el], b[(self.g + self.n) * el:]
        return bool((head == CANARY).all()) and bool((tail == CANARY).all())


def test_no_call_writes_outside_its_buffers():
    B, Hq, Hkv, N, K, Qn, C = 2, 8, 2, 70, 16, 5, 4
    d = lsk.make_dims(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, max_blocks=N, budget_blocks=K, n_queries=Qn,
                      fetch_cap=C)
    g = torch.Generator()
    g.manual_seed(5)
    kv = (torch.randn(B, Hkv, N, 2, 16, 128, generator=g) * 2).to(torch.bfloat16)
    ctx0 = torch.tensor([N * 16 - 5, 40 * 16 + 3], dtype=torch.int32)
    bufs = {
        "host_kv": Guarded((B, Hkv, N, 2, 16, 128), torch.bfloat16, "pinned", kv),
        "ctx": Guarded((B,), torch.int32, init=ctx0),
        "ctx_out": Guarded((B,), torch.int32, init=ctx0),
        "kmin": Guarded((B, Hkv, N, 128), torch.bfloat16, init=torch.zeros(B, Hkv, N, 128)),
        "kmax": Guarded((B, Hkv, N, 128), torch.bfloat16, init=torch.zeros(B, Hkv, N, 128)),
        "scores": Guarded((B, Hkv, N), torch.float32, init=torch.zeros(B, Hkv, N)),
        "sel": Guarded((B, Hkv, K), torch.int32, init=torch.full((B, Hkv, K), -1)),
        "sel_score": Guarded((B, Hkv, K), torch.float32, init=torch.zeros(B, Hkv, K)),
        "exact": Guarded((B, Hkv, K), torch.int32, init=torch.full((B, Hkv, K), -1)),
        "slot_table": Guarded((B, Hkv, K), torch.int32, init=torch.full((B, Hkv, K), -1)),
        "last_used": Guarded((B, Hkv, K), torch.int32, init=torch.full((B, Hkv, K), -1)),
        "fetch_slot": Guarded((B, Hkv, C), torch.int32, init=torch.full((B, Hkv, C), -1)),
        "fetch_block": Guarded((B, Hkv, C), torch.int32, init=torch.full((B, Hkv, C), -1)),
        "n_fetch": Guarded((B, Hkv), torch.int32, init=torch.zeros(B, Hkv)),
        "count": Guarded((B, Hkv), torch.int32, init=torch.zeros(B, Hkv)),
        "pool": Guarded((B, Hkv, K, 2, 16, 128), torch.bfloat16, init=torch.zeros(B, Hkv, K, 2, 16, 128)),
        "out": Guarded((B, Qn, Hq, 128), torch.float32, init=torch.zeros(B, Qn, Hq, 128)),
        "lse": Guarded((B, Qn, Hq), torch.float32, init=torch.zeros(B, Qn, Hq)),
        "ws": Guarded((lsk.workspace_bytes(d),), torch.uint8, init=torch.zeros(lsk.workspace_bytes(d))),
        "step": Guarded((4,), torch.int32, init=torch.zeros(4)),
        "mask": Guarded((B, Hkv, K), torch.uint8, init=torch.zeros(B, Hkv, K)),
    }
    t = {k: v.t for k, v in bufs.items()}
    scale = 1 / math.sqrt(128)
    qs = [(torch.randn(B, Qn, Hq, 128, generator=g)).to(torch.bfloat16).to(DEV) for _ in range(8)]

    lsk.build_summaries(d, t["host_kv"], t["ctx"], t["kmin"], t["kmax"])
    lsk.score_select(d, qs[0], t["kmin"], t["kmax"], t["ctx"], t["sel"], t["sel_score"], t["ws"])
    lsk.plan_fetch(d, t["sel"], t["slot_table"], t["last_used"], 0, t["fetch_slot"], t["fetch_block"], t["n_fetch"])
    lsk.prefetch(d, t["host_kv"], t["fetch_slot"], t["fetch_block"], t["n_fetch"], t["pool"])
    # scores + top-K + plan in one launch, LRU (scores in the workspace) and score-ordered victims
    lsk.score_select_plan(d, qs[0], t["kmin"], t["kmax"], t["ctx"], t["sel"], t["sel_score"], None, t["slot_table"],
                          t["last_used"], 0, None, t["fetch_slot"], t["fetch_block"], t["n_fetch"], t["ws"])
    lsk.score_select_plan(d, qs[0], t["kmin"], t["kmax"], t["ctx"], t["sel"], None, t["scores"], t["slot_table"],
                          t["last_used"], 0, t["step"], t["fetch_slot"], t["fetch_block"], t["n_fetch"], t["ws"])
    for step in range(1, 4):
        q = qs[step]
        lsk.sparse_attn(d, q, t["pool"], t["slot_table"], t["ctx"], scale, t["out"], t["lse"], t["ws"])
        lsk.lookahead_scores(d, q, t["kmin"], t["kmax"], t["ctx"], t["scores"])
        lsk.select_topk(d, t["scores"], t["ctx"], t["sel"], t["sel_score"])
        lsk.plan_fetch_scored(d, t["sel"], t["scores"], t["slot_table"], t["last_used"], step, t["fetch_slot"],
                              t["fetch_block"], t["n_fetch"])
        lsk.prefetch(d, t["host_kv"], t["fetch_slot"], t["fetch_block"], t["n_fetch"], t["pool"])
        lsk.score_select_rows(d, q, 0, 1, t["kmin"], t["kmax"], t["ctx"], t["exact"], None, t["ws"])
        lsk.block_overlap(d, t["sel"], t["exact"], t["count"])
        t["mask"].copy_((torch.rand(B, Hkv, K, generator=g) < 0.25).to(torch.uint8))
        lsk.evict_slots(d, t["mask"], t["slot_table"])
        k_new, v_new = W.append_rows(W.WORKLOADS["llama8b_32k"].with_(batch=B, n_kv_heads=Hkv), 0, step)
        lsk.append_kv(d, k_new.to(DEV), v_new.to(DEV), t["ctx"], t["ctx_out"], t["host_kv"], t["kmin"], t["kmax"],
                      t["slot_table"], t["pool"])
        t["ctx"].copy_(t["ctx_out"])
    # the native layer step, plans numbered on the device, on one stream
    s = torch.cuda.current_stream()
    evs = [torch.cuda.Event() for _ in range(3)]
    for ev in evs:
        ev.record(s)
    layer = lsk.make_layer(d, t["host_kv"], t["kmin"], t["kmax"], t["pool"], t["slot_table"], t["last_used"],
                           t["sel"], t["sel_score"], None, t["fetch_slot"], t["fetch_block"], t["n_fetch"], t["out"],
                           t["lse"])
    sync = lsk.StepSync(s.cuda_stream, s.cuda_stream, evs[0].cuda_event, evs[1].cuda_event, 0)
    t["step"].fill_(4)
    for step in range(4, 7):
        lsk.step_advance(t["step"])
        lsk.decode_layer_step(d, layer, qs[step], t["ctx"], t["mask"], 0, t["step"], scale, t["ws"], sync)
    torch.cuda.synchronize()
    assert lsk.read_device_error(clear=True) == 0
    broken = [name for name, b in bufs.items() if not b.intact()]
    assert not broken, f"writes outside the buffer: {broken}"
    # the calls did write inside: the pool holds fetched blocks and attention has output
    assert int((t["slot_table"] >= 0).sum()) > 0 and bool(torch.isfinite(t["lse"]).any())
