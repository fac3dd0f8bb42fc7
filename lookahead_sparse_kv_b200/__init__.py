"""Python binding of liboasis.so, the B200 lookahead sparse-KV decode path.

Argument marshalling only: every function here forwards torch tensors (or raw
device / host addresses) to the C ABI declared in ``include/oasis.h`` and
raises ``OasisError`` on a non-zero return.  No computation happens in
Python and there is no fallback: if the library is not built, the first call
raises.

The C ABI sees plain pointers, so it cannot tell a short buffer from a long
one.  Before a call, each tensor argument is checked against the dims: its
dtype, that it is contiguous, that it holds at least the elements the call
touches, and that device buffers are on a CUDA device.  A failed check raises
``OasisError`` (EINVAL) before anything is enqueued.  Raw integer addresses
are passed through unchecked: they are the caller's responsibility.  Where
host KV lives (device memory or mapped pinned host memory) is checked by the
library itself.

The operations follow the page "OasisKV: Scaling In-Decode KV Cache Beyond
HBM with Lookahead Sparse Prefetching" (Figures 7-9, Table 2); see the header
for the exact contract of each call.
"""

from __future__ import annotations

import ctypes
import os
import re

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "liboasis.so")
HEADER = os.path.join(os.path.dirname(PKG_DIR), "include", "oasis.h")

OK, EINVAL, ENOTMAPPED, ECUDA, ERANGE = 0, -1, -2, -3, -4
DEVERR_ID_RANGE, DEVERR_TIMEOUT, DEVERR_APPEND_FULL, DEVERR_DUPLICATE = 0x1, 0x2, 0x4, 0x8
HEAD_DIM, BLOCK_TOKENS = 128, 16


class OasisError(RuntimeError):
    def __init__(self, code: int, what: str, msg: str):
        super().__init__(f"{what} failed ({code}): {msg}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in (
        "batch", "n_q_heads", "n_kv_heads", "head_dim", "block_tokens",
        "max_blocks", "budget_blocks", "n_queries", "fetch_cap")]

    def __repr__(self):
        return "Dims(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


def make_dims(batch, n_q_heads, n_kv_heads, max_blocks, budget_blocks, n_queries, fetch_cap,
              head_dim=HEAD_DIM, block_tokens=BLOCK_TOKENS) -> Dims:
    return Dims(batch, n_q_heads, n_kv_heads, head_dim, block_tokens, max_blocks,
                budget_blocks, n_queries, fetch_cap)


def dims_for(w) -> Dims:
    """Dims of a ``workloads.Workload``."""
    return make_dims(w.batch, w.n_q_heads, w.n_kv_heads, w.max_blocks, w.budget_blocks,
                     w.n_queries, w.fetch_cap, w.head_dim, w.block_tokens)


class Layer(ctypes.Structure):
    """oasis_layer: one attention layer's buffers (device addresses)."""
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "host_kv", "kmin", "kmax", "pool", "slot_table", "last_used", "sel", "sel_score", "scores",
        "fetch_slot", "fetch_block", "n_fetch", "out", "lse")]


class StepSync(ctypes.Structure):
    """oasis_step_sync: streams, this layer's events, graph flag, timing events
    (begin / end of the attention, the fused scores + top-K + plan, the gather)."""
    _fields_ = [("main", ctypes.c_void_p), ("copy", ctypes.c_void_p), ("fetch_done", ctypes.c_void_p),
                ("plan_ready", ctypes.c_void_p), ("in_graph", ctypes.c_int32), ("timing", ctypes.c_void_p * 6)]


_LIB = None
_V = ctypes.c_void_p
_I32 = ctypes.c_int32
_SIGS = {
    "oasis_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(Dims)]),
    "oasis_build_summaries": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _I32, _I32, _V, _V, _V]),
    "oasis_append_kv": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _V, _V, _V, _V, _V, _V, _V, _V]),
    "oasis_lookahead_scores": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _V, _V, _V, _V]),
    "oasis_select_topk": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _V, _V, _V]),
    "oasis_score_select": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _V, _V, _V, _V, _V,
                                          ctypes.c_size_t, _V]),
    "oasis_score_select_noalloc": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _V, _V, _V, _V, _V]),
    "oasis_score_select_rows": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _I32, _I32, _V, _V, _V, _V, _V, _V,
                                               ctypes.c_size_t, _V]),
    "oasis_score_select_plan": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _V, _V, _V, _V, _V, _V, _V, _I32, _V,
                                               _V, _V, _V, _V, ctypes.c_size_t, _V]),
    "oasis_block_overlap": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _V, _V]),
    "oasis_plan_fetch": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _V, _I32, _V, _V, _V, _V]),
    "oasis_plan_fetch_scored": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _V, _V, _I32, _V, _V, _V, _V]),
    "oasis_plan_fetch_at": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _V, _V, _V, _V, _V, _V, _V]),
    "oasis_step_advance": (ctypes.c_int, [_V, _V]),
    "oasis_evict_slots": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _V]),
    "oasis_decode_layer_step": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Layer), _V, _V, _V, _I32, _V,
                                               ctypes.c_float, _V, ctypes.c_size_t, ctypes.POINTER(StepSync)]),
    "oasis_prefetch": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _V, _V, _V, _V]),
    "oasis_sparse_attn": (ctypes.c_int, [ctypes.POINTER(Dims), _V, _V, _V, _V, ctypes.c_float,
                                         _V, _V, _V, ctypes.c_size_t, _V]),
    "oasis_read_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int, _V]),
    "oasis_check_dims": (ctypes.c_int, [ctypes.POINTER(Dims)]),
    "oasis_last_error": (ctypes.c_char_p, []),
    "oasis_version": (ctypes.c_char_p, []),
}


def lib() -> ctypes.CDLL:
    """Load liboasis.so (once).  Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m lookahead_sparse_kv_b200.build` (or __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _LIB = L
    return _LIB


def header_symbols(path: str = HEADER):
    """Names of the entry points declared in the C header."""
    with open(path) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(oasis_\w+)\s*\(", text, re.M)))


def last_error() -> str:
    return lib().oasis_last_error().decode()


_BF16, _I32_T, _F32 = "bfloat16", "int32", "float32"
_U8 = ("uint8", "bool")          # byte masks: torch's bool is one byte holding 0 or 1


def _arg(x, what: str, name: str, dtype, numel: int, device: bool = True, nullable: bool = False):
    """Address of tensor argument `name` after checking it against the call:
    dtype, contiguity, at least `numel` elements, and a CUDA device when
    `device` (host KV may be either; the library checks its mapping)."""
    if x is None:
        if nullable:
            return None
        raise OasisError(EINVAL, what, f"{name} is None")
    if isinstance(x, int):
        return x
    names = (dtype,) if isinstance(dtype, str) else dtype
    if str(x.dtype)[len("torch."):] not in names:
        raise OasisError(EINVAL, what, f"{name} must be {' or '.join(names)}, got {x.dtype}")
    if not x.is_contiguous():
        raise OasisError(EINVAL, what, f"{name} must be contiguous")
    if x.numel() < numel:
        raise OasisError(EINVAL, what, f"{name} holds {x.numel()} elements, the call needs {numel}")
    if device and not x.is_cuda:
        raise OasisError(EINVAL, what, f"{name} must be on a CUDA device, got {x.device}")
    return x.data_ptr()


def _ws(x, what: str):
    """Address and byte size of a workspace tensor (any dtype, on the device)."""
    if isinstance(x, int) or x is None:
        raise OasisError(EINVAL, what, "ws must be a tensor (its size is taken from it)")
    if not x.is_contiguous() or not x.is_cuda:
        raise OasisError(EINVAL, what, "ws must be a contiguous CUDA tensor")
    return x.data_ptr(), x.numel() * x.element_size()


class _Sizes:
    """Element counts of every buffer the calls take, from valid dims."""

    def __init__(self, d, what: str):
        rc = lib().oasis_check_dims(ctypes.byref(d))
        if rc != OK:
            raise OasisError(rc, what, last_error())
        B, Hq, Hkv, N, K = d.batch, d.n_q_heads, d.n_kv_heads, d.max_blocks, d.budget_blocks
        D, P, Qn, C = d.head_dim, d.block_tokens, d.n_queries, d.fetch_cap
        self.what = what
        self.b = B
        self.units = B * Hkv
        self.kv = B * Hkv * N * 2 * P * D          # host KV / pool-shaped blocks [B][Hkv][N][2][P][D]
        self.summary = B * Hkv * N * D             # kmin, kmax
        self.q = B * Qn * Hq * D
        self.row = B * Hkv * D                     # one appended K or V row per (b, h)
        self.scores = B * Hkv * N
        self.k = B * Hkv * K                       # sel, sel_score, slot_table, last_used, masks
        self.c = B * Hkv * C                       # fetch_slot, fetch_block
        self.cap = C
        self.pool = B * Hkv * K * 2 * P * D
        self.out = B * Qn * Hq * D
        self.lse = B * Qn * Hq

    def fetch_list(self, x, name):
        return _arg(x, self.what, name, _I32_T, self.c, nullable=self.cap == 0)


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, what: str):
    if rc != OK:
        raise OasisError(rc, what, last_error())


def check_dims(d: Dims) -> int:
    return lib().oasis_check_dims(ctypes.byref(d))


def workspace_bytes(d: Dims) -> int:
    return lib().oasis_workspace_bytes(ctypes.byref(d))


def build_summaries(d, kv, ctx_len, kmin, kmax, first_block=0, n_blocks=None, stream=None):
    w = "oasis_build_summaries"
    z = _Sizes(d, w)
    n = d.max_blocks - first_block if n_blocks is None else n_blocks
    _check(lib().oasis_build_summaries(ctypes.byref(d), _arg(kv, w, "kv", _BF16, z.kv, device=False),
                                       _arg(ctx_len, w, "ctx_len", _I32_T, z.b), first_block, n,
                                       _arg(kmin, w, "kmin", _BF16, z.summary),
                                       _arg(kmax, w, "kmax", _BF16, z.summary), _stream(stream)), w)


def append_kv(d, k_new, v_new, ctx_len, ctx_len_out, host_kv, kmin, kmax, slot_table, pool, stream=None):
    w = "oasis_append_kv"
    z = _Sizes(d, w)
    _check(lib().oasis_append_kv(ctypes.byref(d), _arg(k_new, w, "k_new", _BF16, z.row),
                                 _arg(v_new, w, "v_new", _BF16, z.row), _arg(ctx_len, w, "ctx_len", _I32_T, z.b),
                                 _arg(ctx_len_out, w, "ctx_len_out", _I32_T, z.b, nullable=True),
                                 _arg(host_kv, w, "host_kv", _BF16, z.kv, device=False, nullable=True),
                                 _arg(kmin, w, "kmin", _BF16, z.summary), _arg(kmax, w, "kmax", _BF16, z.summary),
                                 _arg(slot_table, w, "slot_table", _I32_T, z.k, nullable=True),
                                 _arg(pool, w, "pool", _BF16, z.pool, nullable=True),
                                 _stream(stream)), w)


def lookahead_scores(d, q, kmin, kmax, ctx_len, scores, stream=None):
    w = "oasis_lookahead_scores"
    z = _Sizes(d, w)
    _check(lib().oasis_lookahead_scores(ctypes.byref(d), _arg(q, w, "q", _BF16, z.q),
                                        _arg(kmin, w, "kmin", _BF16, z.summary),
                                        _arg(kmax, w, "kmax", _BF16, z.summary),
                                        _arg(ctx_len, w, "ctx_len", _I32_T, z.b),
                                        _arg(scores, w, "scores", _F32, z.scores), _stream(stream)), w)


def select_topk(d, scores, ctx_len, sel, sel_score=None, stream=None):
    w = "oasis_select_topk"
    z = _Sizes(d, w)
    _check(lib().oasis_select_topk(ctypes.byref(d), _arg(scores, w, "scores", _F32, z.scores),
                                   _arg(ctx_len, w, "ctx_len", _I32_T, z.b), _arg(sel, w, "sel", _I32_T, z.k),
                                   _arg(sel_score, w, "sel_score", _F32, z.k, nullable=True), _stream(stream)), w)


def score_select(d, q, kmin, kmax, ctx_len, sel, sel_score, ws, stream=None):
    w = "oasis_score_select"
    z = _Sizes(d, w)
    _check(lib().oasis_score_select(ctypes.byref(d), _arg(q, w, "q", _BF16, z.q),
                                    _arg(kmin, w, "kmin", _BF16, z.summary), _arg(kmax, w, "kmax", _BF16, z.summary),
                                    _arg(ctx_len, w, "ctx_len", _I32_T, z.b), _arg(sel, w, "sel", _I32_T, z.k),
                                    _arg(sel_score, w, "sel_score", _F32, z.k, nullable=True), *_ws(ws, w),
                                    _stream(stream)), w)


def score_select_rows(d, q, row_begin, row_count, kmin, kmax, ctx_len, sel, sel_score, ws, stream=None):
    """Top-K for query rows [row_begin, row_begin + row_count); (0, 1) is the
    verification query alone (exact set / previous-token prediction)."""
    w = "oasis_score_select_rows"
    z = _Sizes(d, w)
    _check(lib().oasis_score_select_rows(ctypes.byref(d), _arg(q, w, "q", _BF16, z.q), row_begin, row_count,
                                         _arg(kmin, w, "kmin", _BF16, z.summary),
                                         _arg(kmax, w, "kmax", _BF16, z.summary),
                                         _arg(ctx_len, w, "ctx_len", _I32_T, z.b), _arg(sel, w, "sel", _I32_T, z.k),
                                         _arg(sel_score, w, "sel_score", _F32, z.k, nullable=True), *_ws(ws, w),
                                         _stream(stream)), w)


def score_select_plan(d, q, kmin, kmax, ctx_len, sel, sel_score, scores, slot_table, last_used, step, step_dev,
                      fetch_slot, fetch_block, n_fetch, ws, stream=None):
    """Scores, top-K and the capped plan in one launch.  scores: None keeps the
    block scores in the workspace (LRU victims), else fp32 [B][Hkv][N] that
    receives them (score-ordered victims); step_dev: None uses ``step``, else an
    int32 device tensor whose first element is read on the device."""
    w = "oasis_score_select_plan"
    z = _Sizes(d, w)
    _check(lib().oasis_score_select_plan(ctypes.byref(d), _arg(q, w, "q", _BF16, z.q),
                                         _arg(kmin, w, "kmin", _BF16, z.summary),
                                         _arg(kmax, w, "kmax", _BF16, z.summary),
                                         _arg(ctx_len, w, "ctx_len", _I32_T, z.b), _arg(sel, w, "sel", _I32_T, z.k),
                                         _arg(sel_score, w, "sel_score", _F32, z.k, nullable=True),
                                         _arg(scores, w, "scores", _F32, z.scores, nullable=True),
                                         _arg(slot_table, w, "slot_table", _I32_T, z.k),
                                         _arg(last_used, w, "last_used", _I32_T, z.k), int(step),
                                         _arg(step_dev, w, "step_dev", _I32_T, 1, nullable=True),
                                         z.fetch_list(fetch_slot, "fetch_slot"),
                                         z.fetch_list(fetch_block, "fetch_block"),
                                         _arg(n_fetch, w, "n_fetch", _I32_T, z.units), *_ws(ws, w),
                                         _stream(stream)), w)


def block_overlap(d, a, b, count, stream=None):
    """count[b][h] = distinct ids of list b also in list a (int32 [B][Hkv][K] each)."""
    w = "oasis_block_overlap"
    z = _Sizes(d, w)
    _check(lib().oasis_block_overlap(ctypes.byref(d), _arg(a, w, "a", _I32_T, z.k), _arg(b, w, "b", _I32_T, z.k),
                                     _arg(count, w, "count", _I32_T, z.units), _stream(stream)), w)


def score_select_noalloc(d, q, kmin, kmax, ctx_len, sel, sel_score=None, stream=None):
    """oasis_score_select without a workspace: for callers that cannot
    allocate or pass device scratch; the scores live in a fixed 4 MiB array
    inside the library (see include/oasis.h for the limit and sharing rules)."""
    w = "oasis_score_select_noalloc"
    z = _Sizes(d, w)
    _check(lib().oasis_score_select_noalloc(ctypes.byref(d), _arg(q, w, "q", _BF16, z.q),
                                            _arg(kmin, w, "kmin", _BF16, z.summary),
                                            _arg(kmax, w, "kmax", _BF16, z.summary),
                                            _arg(ctx_len, w, "ctx_len", _I32_T, z.b), _arg(sel, w, "sel", _I32_T, z.k),
                                            _arg(sel_score, w, "sel_score", _F32, z.k, nullable=True),
                                            _stream(stream)), w)


def plan_fetch(d, sel, slot_table, last_used, step, fetch_slot, fetch_block, n_fetch, stream=None):
    w = "oasis_plan_fetch"
    z = _Sizes(d, w)
    _check(lib().oasis_plan_fetch(ctypes.byref(d), _arg(sel, w, "sel", _I32_T, z.k),
                                  _arg(slot_table, w, "slot_table", _I32_T, z.k),
                                  _arg(last_used, w, "last_used", _I32_T, z.k), int(step),
                                  z.fetch_list(fetch_slot, "fetch_slot"), z.fetch_list(fetch_block, "fetch_block"),
                                  _arg(n_fetch, w, "n_fetch", _I32_T, z.units), _stream(stream)), w)


def plan_fetch_scored(d, sel, scores, slot_table, last_used, step, fetch_slot, fetch_block, n_fetch, stream=None):
    """oasis_plan_fetch with victims ordered by their block's score (lowest first)."""
    w = "oasis_plan_fetch_scored"
    z = _Sizes(d, w)
    _check(lib().oasis_plan_fetch_scored(ctypes.byref(d), _arg(sel, w, "sel", _I32_T, z.k),
                                         _arg(scores, w, "scores", _F32, z.scores),
                                         _arg(slot_table, w, "slot_table", _I32_T, z.k),
                                         _arg(last_used, w, "last_used", _I32_T, z.k), int(step),
                                         z.fetch_list(fetch_slot, "fetch_slot"),
                                         z.fetch_list(fetch_block, "fetch_block"),
                                         _arg(n_fetch, w, "n_fetch", _I32_T, z.units), _stream(stream)), w)


def plan_fetch_at(d, sel, scores, slot_table, last_used, step, fetch_slot, fetch_block, n_fetch, stream=None):
    """Plan with the step number read on the device from ``step`` (int32
    tensor); LRU victims when ``scores`` is None, score-ordered otherwise."""
    w = "oasis_plan_fetch_at"
    z = _Sizes(d, w)
    _check(lib().oasis_plan_fetch_at(ctypes.byref(d), _arg(sel, w, "sel", _I32_T, z.k),
                                     _arg(scores, w, "scores", _F32, z.scores, nullable=True),
                                     _arg(slot_table, w, "slot_table", _I32_T, z.k),
                                     _arg(last_used, w, "last_used", _I32_T, z.k), _arg(step, w, "step", _I32_T, 1),
                                     z.fetch_list(fetch_slot, "fetch_slot"), z.fetch_list(fetch_block, "fetch_block"),
                                     _arg(n_fetch, w, "n_fetch", _I32_T, z.units), _stream(stream)), w)


def evict_slots(d, mask, slot_table, stream=None):
    """Frees the slots whose mask byte (uint8 [B][Hkv][K]) is set."""
    w = "oasis_evict_slots"
    z = _Sizes(d, w)
    _check(lib().oasis_evict_slots(ctypes.byref(d), _arg(mask, w, "mask", _U8, z.k),
                                   _arg(slot_table, w, "slot_table", _I32_T, z.k), _stream(stream)), w)


def make_layer(d, host_kv, kmin, kmax, pool, slot_table, last_used, sel, sel_score, scores, fetch_slot,
               fetch_block, n_fetch, out, lse) -> Layer:
    """oasis_layer from tensors checked against dims `d` (None for the
    nullable sel_score / scores)."""
    w = "make_layer"
    z = _Sizes(d, w)
    return Layer(_arg(host_kv, w, "host_kv", _BF16, z.kv, device=False), _arg(kmin, w, "kmin", _BF16, z.summary),
                 _arg(kmax, w, "kmax", _BF16, z.summary), _arg(pool, w, "pool", _BF16, z.pool),
                 _arg(slot_table, w, "slot_table", _I32_T, z.k), _arg(last_used, w, "last_used", _I32_T, z.k),
                 _arg(sel, w, "sel", _I32_T, z.k), _arg(sel_score, w, "sel_score", _F32, z.k, nullable=True),
                 _arg(scores, w, "scores", _F32, z.scores, nullable=True), z.fetch_list(fetch_slot, "fetch_slot"),
                 z.fetch_list(fetch_block, "fetch_block"), _arg(n_fetch, w, "n_fetch", _I32_T, z.units),
                 _arg(out, w, "out", _F32, z.out), _arg(lse, w, "lse", _F32, z.lse))


def decode_layer_step(d, layer: Layer, q, ctx_len, evict_mask, step, step_dev, scale, ws, sync: StepSync):
    """One layer's decode step (attention, [loss], scores + top-K + plan in one launch, gather) in one call;
    `layer` comes from make_layer, which checked its buffers."""
    w = "oasis_decode_layer_step"
    z = _Sizes(d, w)
    _check(lib().oasis_decode_layer_step(ctypes.byref(d), ctypes.byref(layer), _arg(q, w, "q", _BF16, z.q),
                                         _arg(ctx_len, w, "ctx_len", _I32_T, z.b),
                                         _arg(evict_mask, w, "evict_mask", _U8, z.k, nullable=True), int(step),
                                         _arg(step_dev, w, "step_dev", _I32_T, 1, nullable=True), float(scale),
                                         *_ws(ws, w), ctypes.byref(sync)), w)


def step_advance(step, stream=None):
    """step[0] += 1 on the device, in stream order."""
    w = "oasis_step_advance"
    _check(lib().oasis_step_advance(_arg(step, w, "step", _I32_T, 1), _stream(stream)), w)


def prefetch(d, host_kv, fetch_slot, fetch_block, n_fetch, pool, stream=None):
    w = "oasis_prefetch"
    z = _Sizes(d, w)
    _check(lib().oasis_prefetch(ctypes.byref(d), _arg(host_kv, w, "host_kv", _BF16, z.kv, device=False),
                                z.fetch_list(fetch_slot, "fetch_slot"), z.fetch_list(fetch_block, "fetch_block"),
                                _arg(n_fetch, w, "n_fetch", _I32_T, z.units), _arg(pool, w, "pool", _BF16, z.pool),
                                _stream(stream)), w)


def sparse_attn(d, q, pool, slot_table, ctx_len, scale, out, lse, ws, stream=None):
    w = "oasis_sparse_attn"
    z = _Sizes(d, w)
    _check(lib().oasis_sparse_attn(ctypes.byref(d), _arg(q, w, "q", _BF16, z.q), _arg(pool, w, "pool", _BF16, z.pool),
                                   _arg(slot_table, w, "slot_table", _I32_T, z.k),
                                   _arg(ctx_len, w, "ctx_len", _I32_T, z.b), float(scale),
                                   _arg(out, w, "out", _F32, z.out), _arg(lse, w, "lse", _F32, z.lse), *_ws(ws, w),
                                   _stream(stream)), w)


def read_device_error(clear: bool = True, stream=None) -> int:
    v = ctypes.c_uint32(0)
    _check(lib().oasis_read_device_error(ctypes.byref(v), int(clear), _stream(stream)),
           "oasis_read_device_error")
    return v.value
