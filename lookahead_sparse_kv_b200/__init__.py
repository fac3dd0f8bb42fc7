"""Python binding of liboasis.so, the B200 lookahead sparse-KV decode path.

Argument marshalling only: every function here forwards torch tensors (or raw
device / host addresses) to the C ABI declared in ``include/oasis.h`` and
raises ``OasisError`` on a non-zero return.  No computation happens in
Python and there is no fallback: if the library is not built, the first call
raises.

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
    """oasis_step_sync: streams, this layer's events, graph flag, timing events."""
    _fields_ = [("main", ctypes.c_void_p), ("score", ctypes.c_void_p), ("copy", ctypes.c_void_p),
                ("fetch_done", ctypes.c_void_p), ("plan_ready", ctypes.c_void_p), ("sel_ready", ctypes.c_void_p),
                ("fork", ctypes.c_void_p), ("in_graph", ctypes.c_int32), ("timing", ctypes.c_void_p * 8)]


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


def _p(x):
    """Address of a tensor / int / None for a void* argument."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


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
    n = d.max_blocks - first_block if n_blocks is None else n_blocks
    _check(lib().oasis_build_summaries(ctypes.byref(d), _p(kv), _p(ctx_len), first_block, n,
                                       _p(kmin), _p(kmax), _stream(stream)), "oasis_build_summaries")


def append_kv(d, k_new, v_new, ctx_len, ctx_len_out, host_kv, kmin, kmax, slot_table, pool, stream=None):
    _check(lib().oasis_append_kv(ctypes.byref(d), _p(k_new), _p(v_new), _p(ctx_len), _p(ctx_len_out),
                                 _p(host_kv), _p(kmin), _p(kmax), _p(slot_table), _p(pool),
                                 _stream(stream)), "oasis_append_kv")


def lookahead_scores(d, q, kmin, kmax, ctx_len, scores, stream=None):
    _check(lib().oasis_lookahead_scores(ctypes.byref(d), _p(q), _p(kmin), _p(kmax), _p(ctx_len),
                                        _p(scores), _stream(stream)), "oasis_lookahead_scores")


def select_topk(d, scores, ctx_len, sel, sel_score=None, stream=None):
    _check(lib().oasis_select_topk(ctypes.byref(d), _p(scores), _p(ctx_len), _p(sel), _p(sel_score),
                                   _stream(stream)), "oasis_select_topk")


def score_select(d, q, kmin, kmax, ctx_len, sel, sel_score, ws, stream=None):
    _check(lib().oasis_score_select(ctypes.byref(d), _p(q), _p(kmin), _p(kmax), _p(ctx_len), _p(sel),
                                    _p(sel_score), _p(ws), ws.numel() * ws.element_size(),
                                    _stream(stream)), "oasis_score_select")


def score_select_rows(d, q, row_begin, row_count, kmin, kmax, ctx_len, sel, sel_score, ws, stream=None):
    """Top-K for query rows [row_begin, row_begin + row_count); (0, 1) is the
    verification query alone (exact set / previous-token prediction)."""
    _check(lib().oasis_score_select_rows(ctypes.byref(d), _p(q), row_begin, row_count, _p(kmin), _p(kmax),
                                         _p(ctx_len), _p(sel), _p(sel_score), _p(ws),
                                         ws.numel() * ws.element_size(), _stream(stream)),
           "oasis_score_select_rows")


def block_overlap(d, a, b, count, stream=None):
    """count[b][h] = distinct ids of list b also in list a (int32 [B][Hkv][K] each)."""
    _check(lib().oasis_block_overlap(ctypes.byref(d), _p(a), _p(b), _p(count), _stream(stream)),
           "oasis_block_overlap")


def score_select_noalloc(d, q, kmin, kmax, ctx_len, sel, sel_score=None, stream=None):
    """oasis_score_select without a workspace: for callers that cannot
    allocate or pass device scratch; the scores live in a fixed 4 MiB array
    inside the library (see include/oasis.h for the limit and sharing rules)."""
    _check(lib().oasis_score_select_noalloc(ctypes.byref(d), _p(q), _p(kmin), _p(kmax), _p(ctx_len), _p(sel),
                                            _p(sel_score), _stream(stream)), "oasis_score_select_noalloc")


def plan_fetch(d, sel, slot_table, last_used, step, fetch_slot, fetch_block, n_fetch, stream=None):
    _check(lib().oasis_plan_fetch(ctypes.byref(d), _p(sel), _p(slot_table), _p(last_used), int(step),
                                  _p(fetch_slot), _p(fetch_block), _p(n_fetch), _stream(stream)),
           "oasis_plan_fetch")


def plan_fetch_scored(d, sel, scores, slot_table, last_used, step, fetch_slot, fetch_block, n_fetch, stream=None):
    """oasis_plan_fetch with victims ordered by their block's score (lowest first)."""
    _check(lib().oasis_plan_fetch_scored(ctypes.byref(d), _p(sel), _p(scores), _p(slot_table), _p(last_used),
                                         int(step), _p(fetch_slot), _p(fetch_block), _p(n_fetch),
                                         _stream(stream)), "oasis_plan_fetch_scored")


def plan_fetch_at(d, sel, scores, slot_table, last_used, step, fetch_slot, fetch_block, n_fetch, stream=None):
    """Plan with the step number read on the device from ``step`` (int32
    tensor); LRU victims when ``scores`` is None, score-ordered otherwise."""
    _check(lib().oasis_plan_fetch_at(ctypes.byref(d), _p(sel), _p(scores), _p(slot_table), _p(last_used), _p(step),
                                     _p(fetch_slot), _p(fetch_block), _p(n_fetch), _stream(stream)),
           "oasis_plan_fetch_at")


def evict_slots(d, mask, slot_table, stream=None):
    """Frees the slots whose mask byte (uint8 [B][Hkv][K]) is set."""
    _check(lib().oasis_evict_slots(ctypes.byref(d), _p(mask), _p(slot_table), _stream(stream)), "oasis_evict_slots")


def make_layer(host_kv, kmin, kmax, pool, slot_table, last_used, sel, sel_score, scores, fetch_slot, fetch_block,
               n_fetch, out, lse) -> Layer:
    """oasis_layer from tensors (None for the nullable sel_score / scores)."""
    return Layer(*[_p(t) for t in (host_kv, kmin, kmax, pool, slot_table, last_used, sel, sel_score, scores,
                                    fetch_slot, fetch_block, n_fetch, out, lse)])


def decode_layer_step(d, layer: Layer, q, ctx_len, evict_mask, step, step_dev, scale, ws, sync: StepSync):
    """One layer's decode step (attention, [loss], scores + top-K, plan, gather) in one call."""
    _check(lib().oasis_decode_layer_step(ctypes.byref(d), ctypes.byref(layer), _p(q), _p(ctx_len), _p(evict_mask),
                                         int(step), _p(step_dev), float(scale), _p(ws),
                                         ws.numel() * ws.element_size(), ctypes.byref(sync)),
           "oasis_decode_layer_step")


def step_advance(step, stream=None):
    """step[0] += 1 on the device, in stream order."""
    _check(lib().oasis_step_advance(_p(step), _stream(stream)), "oasis_step_advance")


def prefetch(d, host_kv, fetch_slot, fetch_block, n_fetch, pool, stream=None):
    _check(lib().oasis_prefetch(ctypes.byref(d), _p(host_kv), _p(fetch_slot), _p(fetch_block),
                                _p(n_fetch), _p(pool), _stream(stream)), "oasis_prefetch")


def sparse_attn(d, q, pool, slot_table, ctx_len, scale, out, lse, ws, stream=None):
    _check(lib().oasis_sparse_attn(ctypes.byref(d), _p(q), _p(pool), _p(slot_table), _p(ctx_len),
                                   float(scale), _p(out), _p(lse), _p(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)), "oasis_sparse_attn")


def read_device_error(clear: bool = True, stream=None) -> int:
    v = ctypes.c_uint32(0)
    _check(lib().oasis_read_device_error(ctypes.byref(v), int(clear), _stream(stream)),
           "oasis_read_device_error")
    return v.value
