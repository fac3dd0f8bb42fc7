"""The C ABI library loads, exports every entry point its header declares, and
rejects bad arguments on the host before touching a device.  CPU only."""

import ctypes
import subprocess

import pytest

import lookahead_sparse_kv_b200 as lsk
from lookahead_sparse_kv_b200 import build as lsk_build


@pytest.fixture(scope="module")
def L():
    lsk_build.build()
    return lsk.lib()


def test_header_symbols_all_exported(L):
    names = lsk.header_symbols()
    assert len(names) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", lsk.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(L, n)


def _good():
    return lsk.make_dims(batch=2, n_q_heads=8, n_kv_heads=2, max_blocks=64, budget_blocks=16,
                         n_queries=5, fetch_cap=4)


def test_check_dims_accepts_pages_shapes(L):
    assert lsk.check_dims(_good()) == lsk.OK
    from lookahead_sparse_kv_b200 import workloads as W
    for w in W.WORKLOADS.values():
        assert lsk.check_dims(lsk.dims_for(w)) == lsk.OK, w.name


@pytest.mark.parametrize("field,value", [
    ("head_dim", 64), ("block_tokens", 32), ("n_q_heads", 7), ("budget_blocks", 0),
    ("budget_blocks", 2048), ("max_blocks", 8), ("fetch_cap", 17), ("fetch_cap", -1),
    ("n_queries", 0), ("n_queries", 17), ("batch", 0), ("max_blocks", 40000),
])
def test_check_dims_rejects(L, field, value):
    d = _good()
    setattr(d, field, value)
    assert lsk.check_dims(d) == lsk.EINVAL
    assert lsk.workspace_bytes(d) == 0
    assert lsk.last_error()


def test_workspace_size_covers_scores_and_partials(L):
    d = _good()
    ws = lsk.workspace_bytes(d)
    rows = d.n_queries * d.group
    assert ws >= 4 * d.batch * d.n_kv_heads * d.max_blocks
    # attention partials: one per chunk of at least 2 tiles of 8 slots (4 tiles above 32 rows)
    tiles = -(-d.budget_blocks // 8)
    min_ct = min(tiles, 2 if rows <= 32 else 4)
    assert ws >= 4 * d.batch * d.n_kv_heads * -(-tiles // min_ct) * rows * 129


def test_null_and_misaligned_pointers_rejected_on_host(L):
    d = _good()
    rc = L.oasis_build_summaries(ctypes.byref(d), None, None, 0, 4, None, None, None)
    assert rc == lsk.EINVAL and "NULL" in lsk.last_error()
    rc = L.oasis_plan_fetch(ctypes.byref(d), 16, 32, 48, 0, 64, 80, 97, None)
    assert rc == lsk.EINVAL and "aligned" in lsk.last_error()
    rc = L.oasis_build_summaries(ctypes.byref(d), 16, 32, 60, 8, 48, 64, None)
    assert rc == lsk.EINVAL and "block range" in lsk.last_error()
    rc = L.oasis_sparse_attn(ctypes.byref(d), 16, 32, 48, 64, 1.0, 80, 96, 112, 10, None)
    assert rc == lsk.EINVAL and "workspace" in lsk.last_error()
    with pytest.raises(lsk.OasisError):
        lsk.plan_fetch(d, None, None, None, 0, None, None, None, stream=0)


def test_version_string(L):
    assert b"sm_100a" in L.oasis_version()


def test_native_layer_step_rejects_missing_streams_and_events(L):
    """oasis_decode_layer_step checks its layer / sync arguments before any
    CUDA call: no sync or no events are EINVAL, and with them given the
    attention's own checks answer for the NULL buffers."""
    d = lsk.make_dims(batch=1, n_q_heads=8, n_kv_heads=2, max_blocks=64, budget_blocks=16, n_queries=5,
                      fetch_cap=4)
    layer = lsk.Layer()

    def call(sync):
        return L.oasis_decode_layer_step(ctypes.byref(d), ctypes.byref(layer), None, None, None, 1, None,
                                         ctypes.c_float(0.1), None, 0, sync)

    assert call(None) == lsk.EINVAL
    s = lsk.StepSync()                                   # NULL streams are the default stream
    assert call(ctypes.byref(s)) == lsk.EINVAL and "events" in lsk.last_error()
    s.fetch_done = s.plan_ready = 2
    s.in_graph = 1                                       # no fetch_done wait: nothing reaches the device
    assert call(ctypes.byref(s)) == lsk.EINVAL and "NULL" in lsk.last_error()


def test_binding_checks_tensors_before_calling():
    """The Python binding rejects a tensor that does not fit the call (dtype,
    layout, size, device) with EINVAL before the library sees a pointer;
    raw integer addresses are passed through unchecked."""
    import torch
    d = _good()
    B, H, K = d.batch, d.n_kv_heads, d.budget_blocks
    good = torch.zeros(B * H * K, dtype=torch.int32)

    def err(fn):
        with pytest.raises(lsk.OasisError) as e:
            fn()
        assert e.value.code == lsk.EINVAL
        return str(e.value)

    # the mask goes in as a raw address (unchecked), so the slot table is the argument under test
    assert "slot_table must be int32" in err(lambda: lsk.evict_slots(d, 16, good.float()))
    assert "slot_table must be contiguous" in err(lambda: lsk.evict_slots(d, 16, good.view(B * H, K).t()))
    assert "slot_table holds" in err(lambda: lsk.evict_slots(d, 16, good[1:]))
    assert "slot_table must be on a CUDA device" in err(lambda: lsk.evict_slots(d, 16, good))
    assert "mask holds" in err(lambda: lsk.evict_slots(d, torch.zeros(B * H * K - 1, dtype=torch.uint8), 16))
    assert "mask is None" in err(lambda: lsk.evict_slots(d, None, good))
    bad = _good()
    bad.head_dim = 64
    assert "head_dim" in err(lambda: lsk.evict_slots(bad, None, None))
    # a raw address skips the tensor checks; the library then answers for it (NULL slot table)
    with pytest.raises(lsk.OasisError) as e:
        lsk.evict_slots(d, 16, 0)
    assert e.value.code == lsk.EINVAL and "slot_table" in str(e.value)


@pytest.mark.parametrize("dims", ["null", "valid"])
def test_every_entry_point_rejects_null_arguments(L, dims):
    """Each int-returning entry point, called with NULL pointers (and NULL or
    valid dims), returns EINVAL with a message: host-side checks come before
    any device work, so this holds on a machine without a GPU."""
    d = _good()
    for name, (res, args) in lsk._SIGS.items():
        if res is not ctypes.c_int or not args or (dims == "valid" and name == "oasis_check_dims"):
            continue                  # (valid dims are all oasis_check_dims takes)
        vals = []
        for a in args:
            if a in (ctypes.c_int32, ctypes.c_int, ctypes.c_size_t):
                vals.append(0)
            elif a is ctypes.c_float:
                vals.append(1.0)
            elif dims == "valid" and a is not None and getattr(a, "_type_", None) is lsk.Dims:
                vals.append(ctypes.byref(d))
            else:
                vals.append(None)
        rc = getattr(L, name)(*vals)
        expect = lsk.EINVAL
        if name == "oasis_score_select_noalloc" and dims == "valid" and not _has_gpu():
            expect = lsk.ECUDA        # it looks up its device-resident scratch first: no device, no scratch
        assert rc == expect, f"{name} returned {rc}"
        assert lsk.last_error(), name


def _has_gpu():
    import torch
    return torch.cuda.is_available()


def test_binding_passes_optional_buffers_through_as_null():
    """Arguments the header documents as optional (here the append's host KV,
    slot table and pool) reach the library as NULL: the error below is the
    library's own host-side check of a required pointer given as a raw NULL
    address, raised before any device work, not the binding's None check."""
    d = _good()
    with pytest.raises(lsk.OasisError) as e:
        lsk.append_kv(d, 16, 32, 48, None, None, 0, 80, None, None)
    assert e.value.code == lsk.EINVAL and "kmin is NULL" in str(e.value)
    with pytest.raises(lsk.OasisError) as e:
        lsk.append_kv(d, 16, 32, 48, None, None, None, 80, None, None)
    assert "kmin is None" in str(e.value)                  # required: the binding stops it
