"""Host-side logic of the benchmark: the kernel-source hash that keeps the
ncu traffic file tied to the kernels it was taken on, and the derived
metrics (overlap efficiency, token-KV intensity).  CPU only."""

import math

import bench
from lookahead_sparse_kv_b200 import workloads as W


def test_strip_comments_keeps_code_and_string_literals():
    src = 'int a = 1; // gone\n/* gone\n too */ asm("ld.global // kept"); const char* s = "a\\"b"; // x'
    out = bench.strip_comments(src)
    assert "gone" not in out and "x" not in out.split()
    assert 'asm("ld.global // kept");' in out
    assert '"a\\"b"' in out
    assert bench.strip_comments("a  \n\n  b") == "a b"


def test_kernel_hash_ignores_comment_edits_only(tmp_path, monkeypatch):
    csrc = tmp_path / "lookahead_sparse_kv_b200" / "csrc"
    csrc.mkdir(parents=True)
    f = csrc / "k.cuh"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f.write_text("__global__ void k(int* p) { p[0] = 1; }  // first\n")
    h1 = bench.kernel_source_hash()
    f.write_text("// a new header comment\n__global__ void k(int* p) {\n    p[0] = 1;  /* reworded */\n}\n")
    assert bench.kernel_source_hash() == h1
    f.write_text("__global__ void k(int* p) { p[0] = 2; }\n")
    assert bench.kernel_source_hash() != h1


def test_overlap_efficiency_bounds():
    iso = {"sparse_attn": 0.03, "score_select_plan": 0.035, "prefetch": 0.25}
    t_c, t_f = 0.065, 0.25                # attention + (scores, top-K and plan)
    full = bench.overlap_efficiency(iso, max(t_c, t_f))          # perfect overlap
    none = bench.overlap_efficiency(iso, t_c + t_f)              # back to back
    assert math.isclose(full["value"], 1.0) and math.isclose(none["value"], 0.0, abs_tol=1e-12)
    assert math.isclose(full["compute_ms"], t_c) and full["fetch_ms"] == t_f


def test_token_kv_intensity_of_the_32k_layer():
    w = W.WORKLOADS["llama8b_32k"]
    r = bench.token_kv_intensity(w, 1583)
    # sparse HBM bytes: 128 units x (128 slots x 8 KiB + 2048 summaries x 512 B) = 256 MiB
    assert math.isclose(r["hbm_tokens_per_mib"], 16 / 256)
    # dense reads the whole 2 GiB of KV
    assert math.isclose(r["dense_hbm_tokens_per_mib"], 16 / 2048)
    assert math.isclose(r["pcie_tokens_per_mib"], 16 / (1583 * 8192 / 2 ** 20))


class _FakeTimer:
    def __init__(self, ms):
        self.ms = ms

    def mean_ms(self, name):
        return self.ms.get(name)


class _FakeLayer:
    def __init__(self, w):
        import torch
        self.out = torch.empty(w.batch, w.n_queries, w.n_q_heads, w.head_dim)
        self.lse = torch.empty(w.batch, w.n_queries, w.n_q_heads)


def test_gpu_line_keeps_the_contract(capsys):
    """The GPU arm's JSON line, built from fake timings: every key of the
    contract, the shared metric/config, and the roofline of the dominant kernel."""
    import argparse
    import json

    import torch
    w = W.WORKLOADS[bench.WORKLOAD]
    nl, steps = 8, 10
    ms_pipe = {"sparse_attn": 0.03, "score_select_plan": 0.04, "prefetch": 0.277}
    res = {
        "w": w, "timer": _FakeTimer(ms_pipe), "layers": [None] * nl,
        "fetch_hist": torch.full((steps * nl,), 1583.0),
        "h2d": {"memcpy_gbs": 55.6, "zero_copy_gbs": 51.1, "peak_gbs": 55.6},
        "iso": {"sparse_attn": 0.03, "score_select_plan": 0.04, "plan_fetch": 0.012, "prefetch": 0.26,
                "select_only": 0.016, "build_summaries": 20.9, "_prefetch_blocks": 1572},
        "ms": 2.25 * steps, "e2e_steps": steps, "e2e_ms": 2.4 * steps, "layer": _FakeLayer(w),
        "reuse": [0.9, 0.89], "host_ms": 2.1 * steps, "host_cost_ms": 0.19,
        "clocks": {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": [], "samples": 10}, "dev_err": 0,
    }
    args = argparse.Namespace(steps=steps, warmup=3, no_cpu_baseline=True)
    bench.emit_gpu(args, res, 1)
    d = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in d, k
    assert d["metric"] == bench.METRIC and d["config"] == bench.headline_config(w, nl, 1)
    assert math.isclose(d["value"], nl / (d["ms_per_step"] * 1e-3))
    assert d["steps"] == steps and d["warmup"] == 3 and d["n_gpus"] == 1 and d["scaling"] == "weak"
    r = d["roofline"]
    assert r["kernel"] == "prefetch" and r["bound"] == "h2d" and r["unit"] == "GB/s" and r["peak"] == 55.6
    assert math.isclose(r["achieved"], 1583 * w.block_bytes / 0.277e-3 / 1e9)
    assert math.isclose(r["frac"], r["achieved"] / r["peak"])
    e = d["e2e"]
    assert e["unit"] == d["unit"] and e["h2d_bytes_per_step"] > nl * 1583 * w.block_bytes
    assert e["d2h_bytes_per_step"] == nl * (w.batch * w.n_queries * w.n_q_heads * (w.head_dim + 1) * 4)
    assert d["gpu_launches"] == bench.launches_per_layer_step(w) * steps * nl
    assert d["host_kv_layers"] == nl and d["cpus_bound"] is None
    assert d["kernels_isolated"]["sparse_attn"]["bound"] == "hbm"


def test_clock_summary_from_sampled_lines():
    """The clocks record of the bench line, from nvidia-smi rows as
    `--format=csv,noheader,nounits` prints them: median and max SM clock, and
    every throttle reason seen Active in any row; malformed rows are skipped."""
    c = bench.ClockSampler(0)
    c.lines = [
        "1965, 1965, 250.31, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "1950, 1965, 612.02, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "1965, 1965, 640.77, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "[N/A], 1965, 600.00, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage",
        "",
    ]
    s = c.summary()
    assert s == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    c.lines = ["1200, 1965, 900.0, 0x8, Active, Not Active, Active, Not Active"]
    assert c.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    c.lines = []
    assert c.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_host_kv_layers_fit_the_node(monkeypatch):
    """Distinct pinned host-KV layers per rank (2 GiB each for the 32K Llama
    layer): all of them when memory allows, fewer on a tight node, never 0,
    and all of them when the host's memory cannot be read."""
    w = W.WORKLOADS["llama8b_32k"]
    gib = 1 << 30
    assert w.batch * w.n_kv_heads * w.max_blocks * w.block_bytes == 2 * gib
    assert bench.host_kv_layers(w, 8, 1, avail=64 * gib) == 8
    assert bench.host_kv_layers(w, 8, 8, avail=1024 * gib) == 8
    assert bench.host_kv_layers(w, 8, 8, avail=100 * gib) == 4          # 12.5 - 4 GiB per rank
    assert bench.host_kv_layers(w, 8, 8, avail=10 * gib) == 1
    monkeypatch.setattr(bench, "_available_host_bytes", lambda: None)
    assert bench.host_kv_layers(w, 8, 8) == 8
    monkeypatch.undo()
    got = bench._available_host_bytes()
    assert got is None or got > 0


def test_workload_state_aliases_host_kv_past_the_distinct_layers(monkeypatch):
    """build_workload_state with fewer distinct host-KV layers than layers:
    only that many pinned buffers are made, layer l holds buffer l mod L, and
    every layer keeps queries of its own (device parts stubbed)."""
    import torch
    pinned = []
    real_empty = torch.empty

    def empty(*a, pin_memory=False, **k):
        t = real_empty(*a, **k)
        if pin_memory:
            pinned.append(t)
        return t

    class Layer:
        def __init__(self, d, host, device):
            self.host_kv = host

    class Pipe:
        def __init__(self, d, states, ctx, scale, device):
            self.states = states

        def build_summaries(self):
            pass

    monkeypatch.setattr(bench, "LayerState", Layer)
    monkeypatch.setattr(bench, "DecodePipeline", Pipe)
    monkeypatch.setattr(bench.torch, "empty", empty)
    monkeypatch.setattr(bench.torch.cuda, "synchronize", lambda *a, **k: None)
    w = W.WORKLOADS["llama8b_32k"].with_(batch=1, n_q_heads=8, n_kv_heads=2, context=256, max_blocks=16,
                                          budget_blocks=8, fetch_cap=2)
    st = bench.build_workload_state(w, 3, device="cpu", n_queries=2, layers=5, host_layers=2)
    hosts = [L.host_kv for L in st["layers"]]
    assert len(pinned) == 2
    assert all(hosts[l] is pinned[l % 2] for l in range(5))
    assert not torch.equal(pinned[0], pinned[1])                       # distinct layers draw distinct KV
    assert len(st["qrings"]) == 5 and not torch.equal(st["qrings"][0][0], st["qrings"][2][0])
    st = bench.build_workload_state(w, 3, device="cpu", n_queries=2, layers=3)
    assert len(pinned) == 5                                            # default: one host KV per layer


def test_cpulist_and_gpu_local_cpus(tmp_path):
    """The CPUs local to a GPU, from a sysfs-shaped tree."""
    assert bench.parse_cpulist("0-3,8,10-11\n") == {0, 1, 2, 3, 8, 10, 11}
    assert bench.parse_cpulist("5") == {5}
    dev = tmp_path / "0000:1b:00.0"
    dev.mkdir()
    (dev / "local_cpulist").write_text("0-27,56-83\n")
    assert bench.gpu_local_cpus(0, 0x1B, 0, str(tmp_path)) == set(range(28)) | set(range(56, 84))
    assert bench.gpu_local_cpus(0, 0x1C, 0, str(tmp_path)) is None


def test_available_host_bytes_reads_meminfo_and_cgroup_limits(tmp_path, monkeypatch):
    """MemAvailable, capped by a cgroup limit less the cgroup's use without
    its reclaimable page cache; an unlimited cgroup does not cap."""
    gib = 1 << 30
    mi = tmp_path / "meminfo"
    mi.write_text(f"MemTotal: {512 * gib // 1024} kB\nMemAvailable:   {400 * gib // 1024} kB\n")
    v2, v1 = tmp_path / "v2", tmp_path / "v1"
    v2.mkdir()
    v1.mkdir()
    monkeypatch.setattr(bench, "MEMINFO", str(mi))
    monkeypatch.setattr(bench, "CGROUP_V2", str(v2))
    monkeypatch.setattr(bench, "CGROUP_V1", str(v1))
    assert bench._available_host_bytes() == 400 * gib                   # no cgroup files
    (v2 / "memory.max").write_text("max\n")
    (v2 / "memory.current").write_text(f"{10 * gib}\n")
    assert bench._available_host_bytes() == 400 * gib                   # unlimited
    (v2 / "memory.max").write_text(f"{64 * gib}\n")
    (v2 / "memory.stat").write_text(f"anon {6 * gib}\ninactive_file {4 * gib}\nactive_file 0\n")
    assert bench._available_host_bytes() == 64 * gib - 6 * gib          # 10 used, 4 of it reclaimable
    (v1 / "memory.limit_in_bytes").write_text(f"{32 * gib}\n")
    (v1 / "memory.usage_in_bytes").write_text(f"{2 * gib}\n")
    assert bench._available_host_bytes() == 30 * gib                    # the tightest limit wins
    monkeypatch.setattr(bench, "MEMINFO", str(tmp_path / "missing"))
    (v1 / "memory.limit_in_bytes").unlink()
    (v2 / "memory.max").unlink()
    assert bench._available_host_bytes() is None
