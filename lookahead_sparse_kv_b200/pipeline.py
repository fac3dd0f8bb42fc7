"""Per-layer device state and the stream / event order of a decode step.

OasisKV: Scaling In-Decode KV Cache Beyond HBM with Lookahead Sparse
Prefetching, Figure 8: at step t each layer's drafts drive the top-K
prediction, the selection and the host-to-HBM copy, and the copy has to
complete before the same layer attends at step t+1; the stages of different
layers overlap.
Figure 7 (right): attention at step t runs over the working set staged at
step t-1.

Streams (all work is in liboasis kernels; this module only orders them):

* main  - [append] -> sparse attention -> [residency loss] -> scores + top-K +
          plan in one launch                            (per layer, in order)
* copy  - host-to-HBM gather, high priority, after the layer's plan; the next
          step's append/attention of that layer waits for it

Scoring follows the attention of its layer on the main stream: the plan
rewrites the slot table the attention reads, and the attention kernel holds
all of every SM's shared memory while it runs, so scoring beside it would
only queue behind it.  The gathers of the layers overlap the compute of the
other layers (Figure 8).

Exact-set mode (OasisKV Figures 4 and 6; prediction misses need corrective
fetches): before a layer's attention at step t the main stream ranks the
blocks for the verification query alone (the exact set E_t), counts how many
of E_t the lookahead selection of step t-1, the previous step's exact set and
the resident slots hold, and - with ``exact="correct"`` - plans and gathers
the missing blocks of E_t with no cap, in stream order before the attention.

Victim order: LRU (OasisKV Table 2) or, with ``victims="score"``, the stale
block with the lowest current lookahead score first; the scores of each
layer then go to a buffer of its own.

Native steps: unless the exact-set stage is on, a layer's decode step is one
call into the library (``oasis_decode_layer_step``), which enqueues the
kernels and does the stream / event order above in C, so the host cost per
layer-step is one call instead of several.

Graph mode (``device_step=True``): the step number lives in device memory
(advanced by a kernel at the start of each step, read by the planner), so a
whole multi-layer decode step can be captured once as a CUDA graph
(``capture``) and replayed (``replay``) with one launch per step.  Inside
the graph all gathers join the main stream at the end, so a replay is
self-contained; the price is that the last layers' gathers no longer overlap
the next step's first layers, which matters little for deep stacks.  Appends and the
exact-set stage take per-step host values and are not captured.

Memory: the full KV of every layer lives in pinned host memory; HBM holds per
layer the per-block summaries (N x 512 B per KV head), the fixed pool of K
slots (8 KiB each) and a few small int tables.  One workspace serves all
layers because the main stream runs the layers' kernels in order.
"""

from __future__ import annotations

import torch

from . import (StepSync, append_kv, block_overlap, build_summaries, decode_layer_step, evict_slots, make_dims,
               make_layer, plan_fetch, plan_fetch_at, prefetch, score_select_plan, score_select_rows, sparse_attn,
               step_advance, workspace_bytes)

HEAD_DIM, BLOCK_TOKENS = 128, 16


class LayerState:
    """Device buffers of one attention layer."""

    def __init__(self, d, host_kv: torch.Tensor, device="cuda"):
        B, H, N, K = d.batch, d.n_kv_heads, d.max_blocks, d.budget_blocks
        C, Qn, Hq, D, P = d.fetch_cap, d.n_queries, d.n_q_heads, HEAD_DIM, BLOCK_TOKENS
        assert host_kv.is_pinned() and host_kv.shape == (B, H, N, 2, P, D)
        self.d = d
        self.host_kv = host_kv
        self.kmin = torch.zeros((B, H, N, D), dtype=torch.bfloat16, device=device)
        self.kmax = torch.zeros((B, H, N, D), dtype=torch.bfloat16, device=device)
        self.pool = torch.zeros((B, H, K, 2, P, D), dtype=torch.bfloat16, device=device)
        self.slot_table = torch.full((B, H, K), -1, dtype=torch.int32, device=device)
        self.last_used = torch.full((B, H, K), -1, dtype=torch.int32, device=device)
        self.sel = torch.full((B, H, K), -1, dtype=torch.int32, device=device)
        self.sel_score = torch.empty((B, H, K), dtype=torch.float32, device=device)
        cap = max(C, 1)
        self.fetch_slot = torch.full((B, H, cap), -1, dtype=torch.int32, device=device)
        self.fetch_block = torch.full((B, H, cap), -1, dtype=torch.int32, device=device)
        self.n_fetch = torch.zeros((B, H), dtype=torch.int32, device=device)
        self.out = torch.zeros((B, Qn, Hq, D), dtype=torch.float32, device=device)
        self.lse = torch.zeros((B, Qn, Hq), dtype=torch.float32, device=device)
        self.plan_ready = torch.cuda.Event()
        self.fetch_done = torch.cuda.Event()
        self.hist = None
        self.scores = None

    def enable_exact(self, steps_cap: int, device="cuda"):
        """Buffers of the exact-set mode: two exact sets (this step's and the
        previous one), uncapped fetch lists, and per decode step t (slot
        (t-1) % steps_cap) int32 [B, Hkv] counts: 0 lookahead agreement,
        1 previous-token agreement, 2 resident coverage, 3 corrective fetches."""
        d = self.d
        B, H, K = d.batch, d.n_kv_heads, d.budget_blocks
        self.exact = [torch.full((B, H, K), -1, dtype=torch.int32, device=device) for _ in range(2)]
        self.cfetch_slot = torch.full((B, H, K), -1, dtype=torch.int32, device=device)
        self.cfetch_block = torch.full((B, H, K), -1, dtype=torch.int32, device=device)
        # each [B, Hkv] slice padded to 16 bytes (the library's pointer alignment)
        self.hist = torch.zeros((4, steps_cap, (B * H + 3) // 4 * 4), dtype=torch.int32, device=device)

    def hist_slot(self, k: int, slot: int) -> torch.Tensor:
        d = self.d
        return self.hist[k, slot, : d.batch * d.n_kv_heads].view(d.batch, d.n_kv_heads)

    def device_bytes(self) -> int:
        ts = [self.kmin, self.kmax, self.pool, self.slot_table, self.last_used, self.sel, self.sel_score,
              self.fetch_slot, self.fetch_block, self.n_fetch, self.out, self.lse]
        return sum(t.numel() * t.element_size() for t in ts)


class DecodePipeline:
    """Drives priming and decode steps over a list of layers."""

    def __init__(self, d, layers, ctx_len: torch.Tensor, scale: float, device="cuda",
                 single_stream: bool = False, exact: str | None = None, steps_cap: int = 256,
                 victims: str = "lru", device_step: bool = False):
        assert exact in (None, "measure", "correct") and victims in ("lru", "score")
        assert not (device_step and exact is not None), "the exact-set stage is not graph-capturable"
        self.d, self.layers, self.scale = d, layers, scale
        self.step_dev = torch.zeros(4, dtype=torch.int32, device=device) if device_step else None
        self.graph = None
        self._step_host = 0
        self.exact = exact
        self.victims = victims
        if victims == "score":
            for L in layers:
                if L.scores is None:
                    L.scores = torch.empty((d.batch, d.n_kv_heads, d.max_blocks), dtype=torch.float32,
                                           device=device)
        self.steps_cap = steps_cap
        if exact is not None:
            # uncapped plan / gather for the corrective fetch, with a workspace of its own
            self.d_full = make_dims(d.batch, d.n_q_heads, d.n_kv_heads, d.max_blocks, d.budget_blocks,
                                    d.n_queries, d.budget_blocks, d.head_dim, d.block_tokens)
            self.ws_exact = torch.zeros(workspace_bytes(d), dtype=torch.uint8, device=device)
            for L in layers:
                L.enable_exact(steps_cap, device)
        self.ctx = [ctx_len, ctx_len.clone()]           # ping-pong when tokens are appended
        self.cur = 0
        self.ws = torch.zeros(workspace_bytes(d), dtype=torch.uint8, device=device)
        # a stream of its own in graph mode: capture cannot start on the default stream
        self.main = torch.cuda.Stream(device) if device_step else torch.cuda.current_stream(device)
        if device_step:
            self.main.wait_stream(torch.cuda.current_stream(device))
        lo, hi = torch.cuda.Stream.priority_range()
        # single_stream: the gathers too run on the main stream (the order a
        # one-stream caller would get; the tests compare the two)
        self.copy_stream = self.main if single_stream else torch.cuda.Stream(device, priority=hi)
        # the native step takes raw event handles: create every event now (torch creates them
        # on first record; recording on an idle stream completes at once)
        for L in layers:
            for ev in (L.plan_ready, L.fetch_done):
                ev.record(self.main)
        self._native = [None] * len(layers)
        self.timer = None        # optional: begin(name, stream) / end(name, stream) around each call

    def _t(self, which, name, stream):
        if self.timer is not None:
            getattr(self.timer, which)(name, stream)

    @property
    def ctx_len(self) -> torch.Tensor:
        return self.ctx[self.cur]

    def build_summaries(self):
        for L in self.layers:
            build_summaries(self.d, L.host_kv, self.ctx_len, L.kmin, L.kmax, stream=self.main)

    def _plan(self, d, sel, scores, L, step, fetch_slot, fetch_block, n_fetch):
        if self.step_dev is not None:
            plan_fetch_at(d, sel, scores, L.slot_table, L.last_used, self.step_dev, fetch_slot, fetch_block,
                          n_fetch, stream=self.main)
        else:
            plan_fetch(d, sel, L.slot_table, L.last_used, step, fetch_slot, fetch_block, n_fetch, stream=self.main)

    def _select_plan_fetch(self, i, L, q, step, ctx):
        d, main = self.d, self.main
        self._t("begin", "score_select_plan", main)
        score_select_plan(d, q, L.kmin, L.kmax, ctx, L.sel, L.sel_score, L.scores if self.victims == "score" else None,
                          L.slot_table, L.last_used, 0 if step is None else step, self.step_dev, L.fetch_slot,
                          L.fetch_block, L.n_fetch, self.ws, stream=main)
        self._t("end", "score_select_plan", main)
        L.plan_ready.record(main)
        self.copy_stream.wait_event(L.plan_ready)
        self._t("begin", "prefetch", self.copy_stream)
        prefetch(d, L.host_kv, L.fetch_slot, L.fetch_block, L.n_fetch, L.pool, stream=self.copy_stream)
        self._t("end", "prefetch", self.copy_stream)
        L.fetch_done.record(self.copy_stream)

    def _native_layer(self, i, L):
        if self._native[i] is None:
            self._native[i] = make_layer(self.d, L.host_kv, L.kmin, L.kmax, L.pool, L.slot_table, L.last_used, L.sel,
                                         L.sel_score, L.scores if self.victims == "score" else None, L.fetch_slot,
                                         L.fetch_block, L.n_fetch, L.out, L.lse)
        return self._native[i]

    def _native_sync(self, i, L, in_graph):
        sync = StepSync(self.main.cuda_stream, self.copy_stream.cuda_stream, L.fetch_done.cuda_event,
                        L.plan_ready.cuda_event, 1 if in_graph else 0)
        if self.timer is not None and hasattr(self.timer, "native_handles"):
            for k, h in enumerate(self.timer.native_handles()):
                sync.timing[k] = h
        return sync

    def _exact_step(self, L, q, t, ctx):
        """Exact set of step t, agreement counts, optional corrective fetch (main stream)."""
        d, main = self.d, self.main
        cur, prev = L.exact[t % 2], L.exact[(t - 1) % 2]
        h = [L.hist_slot(k, (t - 1) % self.steps_cap) for k in range(4)]
        self._t("begin", "exact_set", main)
        score_select_rows(d, q, 0, 1, L.kmin, L.kmax, ctx, cur, None, self.ws_exact, stream=main)
        block_overlap(d, L.sel, cur, h[0], stream=main)
        if t > 1:
            block_overlap(d, prev, cur, h[1], stream=main)
        block_overlap(d, L.slot_table, cur, h[2], stream=main)
        self._t("end", "exact_set", main)
        if self.exact == "correct":
            self._t("begin", "corrective", main)
            self._plan(self.d_full, cur, None, L, t, L.cfetch_slot, L.cfetch_block, h[3])
            prefetch(self.d_full, L.host_kv, L.cfetch_slot, L.cfetch_block, h[3], L.pool, stream=main)
            self._t("end", "corrective", main)

    def prediction_counts(self):
        """Host copies of the per-step counts, int64 [layers, 4, steps_cap, B, Hkv]
        (see LayerState.enable_exact); synchronises."""
        d = self.d
        bh = d.batch * d.n_kv_heads
        h = torch.stack([L.hist[:, :, :bh] for L in self.layers]).cpu().long()
        return h.view(len(self.layers), 4, self.steps_cap, d.batch, d.n_kv_heads)

    def prime(self, q_per_layer):
        """Step 0: select, plan and fetch from the drafts before decoding starts."""
        for i, (L, q) in enumerate(zip(self.layers, q_per_layer)):
            self._select_plan_fetch(i, L, q, None if self.step_dev is not None else 0, self.ctx_len)

    def step(self, t, q_per_layer, appended=None, evict=None, inputs_ready=None, layer_done=None):
        """Decode step t >= 1: per layer [append] -> attention -> [loss] -> select/plan/fetch.

        Each layer's queries are read on the main stream (attention, then
        scores), so queries written there before this call (a non-blocking copy,
        say) are seen by both.
        appended: optional list of (k_new, v_new) per layer, bf16 [B, Hkv, D],
        the token accepted at the previous step; it is written at position
        ctx_len[b] and the context is one token longer from this step on.
        evict: optional list of uint8 masks [B, Hkv, K] per layer; the marked
        slots are freed after the layer's attention (residency loss).
        inputs_ready: optional list of CUDA events, one per layer; layer i's
        work waits for event i first, so a caller can bring each layer's
        queries in on a stream of its own.
        layer_done: optional list of CUDA events, one per layer; event i is
        recorded on the main stream once layer i's attention and plan are
        enqueued (its out and lse are final from there on).
        """
        assert self.graph is None, "a captured pipeline advances by replay()"
        self._step_body(t, q_per_layer, appended, in_graph=False, evict=evict, inputs_ready=inputs_ready,
                        layer_done=layer_done)

    def _step_body(self, t, q_per_layer, appended, in_graph, evict=None, inputs_ready=None, layer_done=None):
        d, main = self.d, self.main
        if self.step_dev is not None:
            if not in_graph:
                assert t == self._step_host + 1, "device-step pipelines take consecutive steps"
                self._step_host = t
            step_advance(self.step_dev, stream=main)
        if appended is None:
            ctx_in = ctx = self.ctx_len
        else:
            ctx_in, ctx = self.ctx[self.cur], self.ctx[1 - self.cur]
        for i, (L, q) in enumerate(zip(self.layers, q_per_layer)):
            if inputs_ready is not None and inputs_ready[i] is not None:
                main.wait_event(inputs_ready[i])
            if not in_graph and (self.exact is not None or appended is not None):
                main.wait_event(L.fetch_done)          # (the native step waits for it itself)
            if appended is not None:
                k_new, v_new = appended[i]
                append_kv(d, k_new, v_new, ctx_in, ctx if i == 0 else None, L.host_kv, L.kmin, L.kmax,
                          L.slot_table, L.pool, stream=main)
            if self.exact is None:
                decode_layer_step(d, self._native_layer(i, L), q, ctx, None if evict is None else evict[i],
                                  0 if t is None else t, self.step_dev, self.scale, self.ws,
                                  self._native_sync(i, L, in_graph))
            else:
                self._exact_step(L, q, t, ctx)
                self._t("begin", "sparse_attn", main)
                sparse_attn(d, q, L.pool, L.slot_table, ctx, self.scale, L.out, L.lse, self.ws, stream=main)
                self._t("end", "sparse_attn", main)
                if evict is not None:
                    evict_slots(d, evict[i], L.slot_table, stream=main)
                self._select_plan_fetch(i, L, q, t, ctx)
            if layer_done is not None and layer_done[i] is not None:
                layer_done[i].record(main)
        if appended is not None:
            self.cur = 1 - self.cur
        if in_graph:
            for L in self.layers:                      # every gather joins before the step ends
                main.wait_event(L.fetch_done)

    def capture(self, q_static, evict_static=None):
        """Captures one decode step over fixed query (and, optionally, loss
        mask) buffers as a CUDA graph (device-step pipelines only, after
        prime()); later steps run by copying their inputs into those buffers
        and calling replay()."""
        assert self.step_dev is not None and self.exact is None and self.timer is None
        self.wait_all()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.main):
            self._step_body(None, q_static, None, in_graph=True, evict=evict_static)
        self.graph = g
        # capture only records the work: the counter is where prime() left it

    def replay(self):
        """One decode step (step counter + every layer), as one graph launch on the main stream."""
        with torch.cuda.stream(self.main):
            self.graph.replay()

    def wait_all(self):
        if self.graph is not None:      # a replay ends with every gather joined to the main stream
            return
        for L in self.layers:
            self.main.wait_event(L.fetch_done)
