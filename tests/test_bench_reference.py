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
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "4", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "layer-steps/s" and d["higher_is_better"] is True
    assert d["steps"] == 4 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["config"] == bench.headline_config(bench.W.WORKLOADS[bench.WORKLOAD], 8, 1)
    assert d["value"] > 0 and d["vs_baseline"] is None and d["scaling"] == "weak"
    # value and ms_per_step describe the same 8-layer step, as on the GPU arm
    assert abs(d["value"] - 8 / (d["ms_per_step"] * 1e-3)) <= 1e-9 * d["value"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_on_nonzero_ranks_prints_nothing():
    env = {**os.environ, "CUDA_VISIBLE_DEVICES": "", "RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2"], cwd=ROOT,
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""
