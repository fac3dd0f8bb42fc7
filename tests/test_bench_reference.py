"""The benchmark's reference arm (the CPU oracle on the host's cores) prints
one JSON line with the headline's metric, unit, direction and config, and
times exactly the requested steps.  CPU only: it needs no GPU."""

import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_line_keeps_the_contract():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "4", "--warmup", "3",
                        "--ref-units", "8"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "layer-steps/s" and d["higher_is_better"] is True
    assert d["steps"] == 4 and d["warmup"] == 3 and d["n_gpus"] == 1
    nl = bench.BENCH_WORKLOADS[bench.WORKLOAD]["layers"]
    assert d["config"] == bench.headline_config(bench.W.WORKLOADS[bench.WORKLOAD], nl, 1)
    assert d["value"] > 0 and d["vs_baseline"] is None and d["scaling"] == "weak"
    # a timed step of this arm is one layer-step of the whole batch: value needs no layer scaling
    assert d["step_layers"] == 1
    assert abs(d["value"] - 1 / (d["ms_per_step"] * 1e-3)) <= 1e-9 * d["value"]
    assert "scaled from 8 to the 128 units" in d["cpu_baseline"]["sample"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_on_nonzero_ranks_prints_nothing():
    env = {**os.environ, "CUDA_VISIBLE_DEVICES": "", "RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2"], cwd=ROOT,
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_cpu_baseline_times_one_core_and_all_cores():
    """The GPU arm's cpu_baseline on a small workload, driven on the CPU:
    a one-core figure, an all-cores figure from spawned processes (one unit
    per usable core), and the host it ran on."""
    from oracle import decode_timing as T
    W = bench.W
    w = W.WORKLOADS["llama8b_32k"].with_(batch=2, n_q_heads=8, n_kv_heads=2, context=1024, max_blocks=64,
                                          budget_blocks=16, fetch_cap=4)

    class _Layer:
        host_kv = W.make_host_kv(w, 0, "cpu")

    qs = W.QueryStream(w, 0, "cpu")
    res = {"layer": _Layer(), "queries": [qs.next() for _ in range(12)]}
    line = bench.cpu_baseline(w, res, n_units=2, fill_steps=2, timed_steps=3, par_fill=1, par_timed=2)
    assert "all_cores_error" not in line, line.get("all_cores_error")
    assert line["kind"] == "oracle" and line["unit"] == "layer-steps/s" and line["value"] > 0
    workers = min(T.usable_cores(), 64, w.batch * w.n_kv_heads)
    assert line["cores"] == workers and line["usable_cores"] == T.usable_cores()
    assert line["single_core"]["cores"] == 1 and line["single_core"]["value"] > 0
    assert line["nproc"] >= 1 and line["cpu_model"]


def test_timing_harness_runs_the_oracles_decode_path():
    """The unit driver the CPU baseline and the reference arm time walks the
    same decode path as the oracle's own multi-step function: after priming
    and 5 steps its slot table, recency and pool are identical."""
    import numpy as np

    import oracle as O
    from oracle import decode_timing as T
    W = bench.W
    w = W.WORKLOADS["llama8b_32k"].with_(batch=1, n_q_heads=4, n_kv_heads=1, context=64 * 16 - 7, max_blocks=64,
                                          budget_blocks=16, fetch_cap=4)
    bits = W.bf16_bits(W.make_host_kv(w, 0, "cpu"))
    qs = W.QueryStream(w, 0, "cpu")
    queries = [O.bf16_bits_to_f64(W.bf16_bits(qs.next())) for _ in range(6)]
    u = T.OracleUnit(bench.oracle_cfg(w), bits)
    u.step(queries[0], 0, attend=False)
    for t in range(1, 6):
        u.step(queries[t], t)
    kv = O.bf16_bits_to_f64(bits)
    keys, vals = kv[:, :, :, 0], kv[:, :, :, 1]
    ctx = np.array([w.context])
    kmin, kmax = O.block_summaries(keys, ctx)
    _, st, lu = O.decode_layer_steps(keys, vals, kmin, kmax, ctx, queries[0], queries[1:], w.budget_blocks,
                                     w.fetch_cap, 1 / np.sqrt(128))
    np.testing.assert_array_equal(u.st, st)
    np.testing.assert_array_equal(u.lu, lu)
    assert (st >= 0).sum() == w.budget_blocks                      # the pool filled up
    for s in range(w.budget_blocks):
        np.testing.assert_array_equal(u.pool_k[0, 0, s], keys[0, 0, st[0, 0, s]])


def test_oracle_worker_pool_fails_fast_and_never_hangs():
    """A worker that dies while setting up, and a pool that outlives its time
    limit, both end in an exception within seconds (the benchmark then
    reports the one-core figure); no process is left behind."""
    import time

    import numpy as np
    import pytest as _pytest

    from oracle import decode_timing as T
    W = bench.W
    w = W.WORKLOADS["llama8b_32k"].with_(batch=1, n_q_heads=4, n_kv_heads=1, context=1024, max_blocks=64,
                                          budget_blocks=16, fetch_cap=4)
    cfg = bench.oracle_cfg(w)
    bits = W.bf16_bits(W.make_host_kv(w, 0, "cpu"))
    qs = W.QueryStream(w, 0, "cpu")
    import oracle as O
    queries = [O.bf16_bits_to_f64(W.bf16_bits(qs.next())) for _ in range(4)]
    t0 = time.monotonic()
    with _pytest.raises(Exception):
        T.run_units_parallel(cfg, [(bits, queries), (np.zeros(3, np.uint16), queries)], 1, 2, 2, timeout_s=60)
    assert time.monotonic() - t0 < 30
    t0 = time.monotonic()
    pool = None
    with _pytest.raises(Exception):
        with T.UnitPool(cfg, [(bits, queries)], 5000, timeout_s=1.0) as pool:  # ≈10 s of set-up: killed at 1 s
            pool.step()
    assert time.monotonic() - t0 < 20
    if pool is not None:
        assert all(p.poll() is not None for p in pool.procs)
