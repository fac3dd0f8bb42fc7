"""Benchmark of the lookahead sparse-KV decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload qwen32b_32k|llama8b_32k]

Default workload (the largest configuration that fits one GPU): a 64-layer
stack shaped like Qwen3-32B at 32K context - batch 16, 64 query / 8 KV
heads, head dim 128, 2,048 blocks of 16 tokens per KV head (about 128 GB of
bf16 KV in pinned host memory), budget 2,048 tokens = 128 blocks, 1
verification + 7 draft queries, fetch cap 16 blocks per head per step, AR(1)
drifting queries, and every step a seeded 10 % of the resident slots lost
from residency before the plan.  Layers beyond the host-KV layers the node
can pin read the host KV of layer l mod that number (the line reports it as
``host_kv_layers``).  ``--workload llama8b_32k`` runs the 8-layer Llama-3.1-8B
stack at 32K (32/8 heads, 1+4 queries) instead.  One step = one decode step
through every layer: per layer, sparse attention over the resident pool,
the residency loss, lookahead scores, top-K selection, the capped fetch plan
and the gather of the missing blocks from pinned host memory, stages of
different layers overlapping as in the OasisKV pipeline (Figure 8).
Metric: layer-steps/s = layers x steps / time (whole job; weak scaling -
every rank runs its own batch, no collective on the data path).

Prints one JSON line (rank 0).  With --impl reference the CPU oracle runs the
same configuration on the host cores (rank 0 only): each timed step is one
decode layer-step of the whole batch.

    python bench.py --prediction [--steps K] [--layers L]

measures prediction quality and the corrective fetch instead (OasisKV
Figures 4 and 6): the same layers with drafts that lead the verification
query, each decode step ranking the blocks for the true query (the exact
set), counting how much of it the lookahead selection and the previous
step's exact set (the previous-token predictor) hold, and - in the third run
- fetching the missing blocks before the attention.  One JSON line.

    python bench.py --ablation [--steps K] [--layers L]

is the synthetic analog of OasisKV Table 2: the fetch cap as a fraction of
the budget K (0.01 .. 0.2 and uncapped) with LRU and score-ordered victims;
per setting the fetch volume, the H2D rate, layer-steps/s and how much of the
exact top-K of the true query and of the lookahead selection is resident.

    python bench.py --longctx [--steps K]

sweeps the 128K long-context stress shape (batch 8, 32/8 heads, 8,192 blocks
per head, heavy-tailed keys, planted blocks that hop every 64 steps) over
budgets of 128 and 256 blocks and caps of 4 / 8 / 16 / 32 blocks per head per
step on 4 pipelined layers, reporting layer-steps/s, H2D GB/s against the
measured PCIe rate and the overlap efficiency of each setting.

    python bench.py --deep [--steps K]

compares the eager stream pipeline with the same decode step captured once as
a CUDA graph and replayed, on a 64-layer stack shaped like Qwen3-32B at 32K
(64/8 heads, 1+7 queries), at batch 16 (transfer-bound) and batch 2 (launch-
bound).  Host KV is shared by layers l and l+8 (8 distinct layers, as the
host-memory fallback allows); queries differ per layer.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import lookahead_sparse_kv_b200 as lsk                                    # noqa: E402
from lookahead_sparse_kv_b200 import workloads as W                        # noqa: E402
from lookahead_sparse_kv_b200.pipeline import DecodePipeline, LayerState  # noqa: E402

WORKLOAD = "qwen32b_32k"            # the default (headline) workload
METRIC = "sparse decode layer-steps/s (score+select+plan+prefetch+attn)"
# per benchmarked workload: default layers, pre-generated query steps, description
BENCH_WORKLOADS = {
    "qwen32b_32k": {"layers": 64, "ring": 16, "host_kv_cap": 16,
                    "desc": "Qwen3-32B-shaped attention layers at 32K context (64/8 heads, 1+7 queries), "
                            "a seeded 10 % residency loss every step, pipelined across layers"},
    "llama8b_32k": {"layers": 8, "ring": 48, "host_kv_cap": 0,
                    "desc": "Llama-3.1-8B-shaped attention layers at 32K context, pipelined across layers"},
}


def data_label(w) -> str:
    loss = f", seeded Bernoulli({w.evict_prob:g}) residency-loss masks" if w.evict_prob > 0 else ""
    return f"synthetic (seeded bf16 KV ~N(0,1) with 4 outlier channels x8, AR(1)-drifting queries{loss})"


def headline_config(w, nl: int, world: int, name: str = WORKLOAD) -> dict:
    """The `config` of the benchmark line, shared by both arms."""
    return {"workload": f"{name}: {nl} {BENCH_WORKLOADS[name]['desc']}",
            "batch": w.batch, "seq_len": w.context, "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads,
            "head_dim": w.head_dim, "block_tokens": w.block_tokens, "budget_blocks": w.budget_blocks,
            "queries": w.n_queries, "fetch_cap": w.fetch_cap, "layers": nl,
            "evict_prob": w.evict_prob,
            "parallelism": f"dp{world} (independent replicas)",
            "l2": "inputs larger than L2: per layer-step 128 MiB summaries + 128 MiB pool read"}
QUERY_RING = 256
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
PROFILES = os.path.join(ROOT, "profiles")


def traffic_path(workload: str) -> str:
    """ncu DRAM bytes per launch for one workload (profiles/traffic_<workload>.json)."""
    return os.path.join(PROFILES, f"traffic_{workload}.json")
KERNELS = ("sparse_attn", "score_select_plan", "prefetch")


# ------------------------------------------------------------------ setup
def ring_index(t: int, n: int) -> int:
    """Index into a ring of n pre-generated query steps walked back and forth,
    so consecutive steps stay consecutive points of the AR(1) path."""
    if n <= 1:
        return 0
    p = t % (2 * n - 2)
    return p if p < n else 2 * n - 2 - p


def rank_workload(rank: int, name: str = WORKLOAD):
    """Weak scaling: every rank runs the benchmarked workload on its own
    seeded batch (no data is exchanged between ranks)."""
    w = W.WORKLOADS[name]
    return w.with_(seed=w.seed + 1000 * rank) if rank else w


def max_over_ranks(x: float) -> float:
    """Max of a per-rank value over all ranks (device time of the slowest
    rank); identity without a process group."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


MEMINFO = "/proc/meminfo"
CGROUP_V2, CGROUP_V1 = "/sys/fs/cgroup", "/sys/fs/cgroup/memory"


def _available_host_bytes():
    """Bytes this process may still take: MemAvailable, capped by the
    container's cgroup memory limit (v2 or v1) when one is set; None if
    neither can be read."""
    vals = []
    try:
        with open(MEMINFO) as f:
            for line in f:
                if line.startswith("MemAvailable:"):
                    vals.append(int(line.split()[1]) * 1024)
    except (OSError, ValueError, IndexError):
        pass
    for base, lim_f, cur_f, cache_key in ((CGROUP_V2, "memory.max", "memory.current", "inactive_file"),
                                          (CGROUP_V1, "memory.limit_in_bytes", "memory.usage_in_bytes",
                                           "total_inactive_file")):
        try:
            with open(os.path.join(base, lim_f)) as f:
                lim = f.read().strip()
            with open(os.path.join(base, cur_f)) as f:
                cur = int(f.read().strip())
            if not (lim.isdigit() and int(lim) < (1 << 60)):
                continue
            cache = 0                                   # reclaimable page cache counts as free
            try:
                with open(os.path.join(base, "memory.stat")) as f:
                    for line in f:
                        k, _, v = line.partition(" ")
                        if k == cache_key:
                            cache = int(v)
            except (OSError, ValueError):
                pass
            vals.append(int(lim) - max(0, cur - cache))
        except (OSError, ValueError):
            pass
    return min(vals) if vals else None


def parse_cpulist(text: str) -> set:
    """CPU numbers of a Linux cpulist string such as "0-31,64-95"."""
    cpus = set()
    for part in text.strip().split(","):
        if not part:
            continue
        lo, _, hi = part.partition("-")
        cpus.update(range(int(lo), int(hi or lo) + 1))
    return cpus


def gpu_local_cpus(domain: int, bus: int, dev: int, sysfs: str = "/sys/bus/pci/devices"):
    """The CPUs the kernel lists as local to the PCI device domain:bus:dev.0
    (its NUMA node's), or None when sysfs does not say."""
    try:
        with open(os.path.join(sysfs, f"{domain:04x}:{bus:02x}:{dev:02x}.0", "local_cpulist")) as f:
            return parse_cpulist(f.read())
    except (OSError, ValueError):
        return None


def bind_near_gpu(device):
    """Restricts this process to the allowed CPUs local to its GPU, so that
    the pinned host KV it allocates next lands in that GPU's NUMA node (first
    touch) and its gathers do not cross the socket interconnect.  Returns the
    number of CPUs kept, or None when nothing was changed."""
    try:
        p = torch.cuda.get_device_properties(device)
        cpus = (gpu_local_cpus(p.pci_domain_id, p.pci_bus_id, p.pci_device_id) or set()) & os.sched_getaffinity(0)
        if not cpus:
            return None
        os.sched_setaffinity(0, cpus)
        return len(cpus)
    except Exception:
        return None


def host_kv_layers(w, layers: int, local_ranks: int, reserve_gib: float = 4.0, avail=None) -> int:
    """Distinct host-KV layers one rank pins: all `layers` when the host's
    available memory holds them for every rank on the node plus a reserve,
    else as many as fit (at least one).  Layer l then reads the host KV of
    layer l mod that number: the same bytes cross PCIe per layer-step, only
    fewer distinct gigabytes sit in host memory."""
    per_layer = w.batch * w.n_kv_heads * w.max_blocks * w.block_bytes
    if avail is None:
        avail = _available_host_bytes()
    if avail is None:
        return layers
    per_rank = avail / max(1, local_ranks) - reserve_gib * (1 << 30)
    return max(1, min(layers, int(per_rank // per_layer)))


def build_workload_state(w, steps: int, device="cuda", n_queries: int | None = None, layers: int = 1,
                         host_layers: int | None = None):
    """Pinned host KV, per-layer device state, pipeline and resident queries
    for `layers` layers of workload `w` (layer l draws its own queries; its KV
    is its own when l < host_layers, else layer l mod host_layers's).  With a
    residency loss (w.evict_prob > 0) each layer also gets a ring of its
    seeded per-step loss masks (uint8 [B, Hkv, K]) as ``mrings``."""
    d = lsk.dims_for(w)
    states, qrings, hosts = [], [], []
    nq = n_queries if n_queries is not None else min(QUERY_RING, max(steps, 1))
    host_layers = layers if host_layers is None else max(1, min(layers, host_layers))
    for l in range(layers):
        if l < host_layers:
            host = torch.empty((w.batch, w.n_kv_heads, w.max_blocks, 2, w.block_tokens, w.head_dim),
                               dtype=torch.bfloat16, pin_memory=True)
            W.make_host_kv(w, layer=l, device=device, out=host)
            torch.cuda.synchronize()
        else:
            host = hosts[l % host_layers]
        states.append(LayerState(d, host, device))
        qs = W.QueryStream(w, l, device)
        qrings.append([qs.next() for _ in range(max(nq, 1))])
        hosts.append(host)
    mrings = None
    if w.evict_prob > 0:
        mrings = [[W.eviction_mask(w, l, i, device).to(torch.uint8) for i in range(max(nq, 1))]
                  for l in range(layers)]
    pipe = DecodePipeline(d, states, W.initial_ctx_len(w, device), 1.0 / math.sqrt(w.head_dim), device)
    pipe.build_summaries()
    torch.cuda.synchronize()
    return {"dims": d, "layers": states, "layer": states[0], "pipe": pipe, "qrings": qrings,
            "queries": qrings[0], "host": hosts[0], "mrings": mrings}


class KernelTimer:
    """CUDA events around each library call, on the stream it runs on."""

    def __init__(self, n):
        self.ev = {k: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in range(n)] for k in KERNELS}
        for pairs in self.ev.values():                 # create them now (torch does on first record),
            for a, b in pairs:                         # not inside the timed region
                a.record()
                b.record()
        self.i = {k: 0 for k in KERNELS}
        self.on = False

    def native_handles(self):
        """Raw begin / end event handles of the next launch of each kernel, in
        the order the native layer step records them (0 = not recorded)."""
        out = []
        for name in KERNELS:
            if self.on and self.i[name] < len(self.ev[name]):
                a, b = self.ev[name][self.i[name]]
                out += [a.cuda_event, b.cuda_event]
                self.i[name] += 1
            else:
                out += [0, 0]
        return out

    def begin(self, name, stream):
        if self.on and self.i[name] < len(self.ev[name]):
            self.ev[name][self.i[name]][0].record(stream)

    def end(self, name, stream):
        if self.on and self.i[name] < len(self.ev[name]):
            self.ev[name][self.i[name]][1].record(stream)
            self.i[name] += 1

    def mean_ms(self, name):
        n = self.i[name]
        if n == 0:
            return None
        return sum(a.elapsed_time(b) for a, b in self.ev[name][:n]) / n


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.proc, self.lines = index, None, []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.index), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# -------------------------------------------------------------- measures
def measure_h2d_peak(device) -> dict:
    """Best of a 1 GiB pinned cudaMemcpyAsync and the zero-copy gather kernel
    over 16K distinct 8 KiB blocks (128 MiB)."""
    n = 1 << 30
    src = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    src.fill_(1)
    dst = torch.empty(n, dtype=torch.uint8, device=device)
    best_copy = 0.0
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src, non_blocking=True)
        b.record()
        b.synchronize()
        best_copy = max(best_copy, n / (a.elapsed_time(b) * 1e-3) / 1e9)
    del dst
    # zero-copy: 128 units x 128 blocks, every entry valid
    d = lsk.make_dims(batch=16, n_q_heads=8, n_kv_heads=8, max_blocks=128, budget_blocks=128,
                      n_queries=1, fetch_cap=128)
    host = src[: 16 * 8 * 128 * 8192].view(torch.bfloat16).view(16, 8, 128, 2, 16, 128)
    pool = torch.empty((16, 8, 128, 2, 16, 128), dtype=torch.bfloat16, device=device)
    ids = torch.arange(128, dtype=torch.int32, device=device).repeat(16, 8, 1).contiguous()
    nf = torch.full((16, 8), 128, dtype=torch.int32, device=device)
    best_zc = 0.0
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        lsk.prefetch(d, host, ids, ids, nf, pool)
        b.record()
        b.synchronize()
        best_zc = max(best_zc, pool.numel() * 2 / (a.elapsed_time(b) * 1e-3) / 1e9)
    return {"memcpy_gbs": best_copy, "zero_copy_gbs": best_zc, "peak_gbs": max(best_copy, best_zc)}


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def strip_comments(src: str) -> str:
    """C/CUDA source without comments and with whitespace collapsed, so that
    a comment edit does not count as a kernel change (string literals kept)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c == '"':                                   # string literal (inline PTX)
            j = i + 1
            while j < n and src[j] != '"':
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash() -> str:
    """Hash of the CUDA sources as the compiler sees them (comments and
    whitespace removed); the ncu traffic file is valid while it matches."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "lookahead_sparse_kv_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(f.encode() + b"\0" + strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def load_traffic(workload: str):
    try:
        with open(traffic_path(workload)) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return {}
    return t.get("kernels", {}) if t.get("source_hash") == kernel_source_hash() else {}


# ------------------------------------------------------------------- run
HOST_COVER_CYCLES = 400_000       # ~0.2 ms of device spin ahead of each isolated launch


def fetch_history(steps: int, layers, device=None):
    """Per-step, per-layer fetch counts of a timed run, in pinned host memory
    filled by asynchronous device-to-host copies on the main stream: a copy
    engine moves them, so no SM kernel runs between the pipeline's own
    launches (a reduction kernel there changed the SMs' shared-memory split
    under the pipeline and cost up to a third of the layer-step rate)."""
    return torch.zeros((steps, len(layers)) + tuple(layers[0].n_fetch.shape), dtype=torch.int32, pin_memory=True)


def record_fetches(hist, i: int, layers):
    for l, L in enumerate(layers):
        hist[i, l].copy_(L.n_fetch, non_blocking=True)


def isolated_kernel_ms(st, reps: int = 20) -> dict:
    """Each library call of one layer-step timed alone on one stream (no
    concurrent kernels), for per-kernel rooflines.  Before every timed launch
    the L2 is flushed (256 MiB written), the device is kept busy while the host
    enqueues, and, when the run has a second layer, the same call runs untimed
    on that layer's buffers: the SMs then enter the timed launch configured
    and with the kernel's code loaded, as after the previous layer's launch in
    the pipeline, while the timed layer's data is still cold."""
    pipe, d = st["pipe"], st["dims"]
    q = st["qrings"][0][0]
    s = torch.cuda.current_stream()
    ctx = pipe.ctx_len

    def layer_calls(L):
        st_c, lu_c = L.slot_table.clone(), L.last_used.clone()
        fs_c, fb_c, nf_c = L.fetch_slot.clone(), L.fetch_block.clone(), L.n_fetch.clone()
        return {
            "sparse_attn": lambda: lsk.sparse_attn(d, q, L.pool, L.slot_table, ctx, pipe.scale, L.out, L.lse, pipe.ws,
                                                   stream=s),
            # the gather of the last plan of the timed run (re-copies the same blocks)
            "prefetch": lambda: lsk.prefetch(d, L.host_kv, L.fetch_slot, L.fetch_block, L.n_fetch, L.pool, stream=s),
            # scores + top-K + plan in one launch, on copies of the slot table and recency
            "score_select_plan": lambda: lsk.score_select_plan(d, q, L.kmin, L.kmax, ctx, L.sel, L.sel_score, None,
                                                               st_c, lu_c, 10 ** 6, None, fs_c, fb_c, nf_c, pipe.ws,
                                                               stream=s),
            "select_only": lambda: lsk.select_topk(d, pipe.ws.view(torch.float32), ctx, L.sel, L.sel_score, stream=s),
            "plan_fetch": lambda: lsk.plan_fetch(d, L.sel, st_c, lu_c, 10 ** 6, fs_c, fb_c, nf_c, stream=s),
            # a1 at admission: summaries of every block from the pinned host KV (rewrites the same values)
            "build_summaries": lambda: lsk.build_summaries(d, L.host_kv, ctx, L.kmin, L.kmax, stream=s),
        }

    L = st["layers"][0]
    calls = layer_calls(L)
    lead = layer_calls(st["layers"][1]) if len(st["layers"]) > 1 else {}
    fetched = int(L.n_fetch.sum().item())
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=q.device)
    out = {}
    torch.cuda.synchronize()
    for name, fn in calls.items():
        tot = 0.0
        n = 3 if name == "build_summaries" else reps          # ~20 ms each: 1 GiB over PCIe
        for _ in range(n):
            flush.zero_()                                  # evict L2 between launches
            # keep the device busy while the host enqueues the calls, so the
            # events time the kernel and not the host's launch work
            torch.cuda._sleep(HOST_COVER_CYCLES)
            if name in lead and name != "build_summaries":
                lead[name]()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(s)
            fn()
            b.record(s)
            b.synchronize()
            tot += a.elapsed_time(b)
        out[name] = tot / n
    out["_prefetch_blocks"] = fetched
    return out


def run_prediction(args, device):
    """Three runs over the same layers of the leading-draft workload: lookahead
    prefetch only, plus the exact-set counts, plus the corrective fetch.  Each
    is primed, warmed up until the pool is full and timed over --steps decode
    steps; the queries are one unbroken AR(1) path (no ring)."""
    w = W.WORKLOADS["llama8b_32k_lead"]
    d = lsk.dims_for(w)
    nl = args.layers
    fill = w.budget_blocks // max(1, w.fetch_cap) + 4          # steps until the pool is full
    total = 1 + fill + args.steps
    layers, qpaths = [], []
    for l in range(nl):
        host = torch.empty((w.batch, w.n_kv_heads, w.max_blocks, 2, w.block_tokens, w.head_dim),
                           dtype=torch.bfloat16, pin_memory=True)
        W.make_host_kv(w, layer=l, device=device, out=host)
        layers.append(LayerState(d, host, device))
        qs = W.QueryStream(w, l, device)
        qpaths.append([qs.next() for _ in range(total)])
    torch.cuda.synchronize()
    ctx = W.initial_ctx_len(w, device)
    out = {}
    for mode in (None, "measure", "correct"):
        for L in layers:
            L.slot_table.fill_(-1)
            L.last_used.fill_(-1)
            L.sel.fill_(-1)
        pipe = DecodePipeline(d, layers, ctx, 1.0 / math.sqrt(w.head_dim), device, exact=mode,
                              steps_cap=total)
        pipe.build_summaries()
        pipe.prime([p[0] for p in qpaths])
        for t in range(1, 1 + fill):
            pipe.step(t, [p[t] for p in qpaths])
        pipe.wait_all()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(pipe.main)
        for t in range(1 + fill, total):
            pipe.step(t, [p[t] for p in qpaths])
        pipe.wait_all()
        e1.record(pipe.main)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        res = {"layer_steps_per_s": nl * args.steps / (ms * 1e-3), "ms_per_step": ms / args.steps}
        if mode is not None:
            c = pipe.prediction_counts()[:, :, fill:total - 1].double()     # timed steps t = fill+1 .. total-1
            k = float(w.budget_blocks)                                      # |exact set| (every context > K blocks)
            per_layer = c.mean(dim=(2, 3, 4)) / k                           # [layers, 4]
            res.update({
                "lookahead_agreement": per_layer[:, 0].mean().item(),
                "previous_token_agreement": per_layer[:, 1].mean().item(),
                "resident_coverage": per_layer[:, 2].mean().item(),
                "lookahead_agreement_per_layer": [round(x, 4) for x in per_layer[:, 0].tolist()],
                "previous_token_agreement_per_layer": [round(x, 4) for x in per_layer[:, 1].tolist()],
            })
            if mode == "correct":
                res["corrective_blocks_per_head_step"] = c[:, 3].mean().item()
                res["corrective_mib_per_layer_step"] = (c[:, 3].sum(dim=(2, 3)).mean().item()
                                                        * w.block_bytes / 2 ** 20)
        out[mode or "lookahead_only"] = res
        del pipe
    # agreement only, on two of the layers, for faster-moving queries: the
    # AR(1) coefficient and drift size set how far the true query moves per step
    sweep = []
    for rho, drift in ((0.9, 0.3), (0.9, 1.0), (0.7, 1.0), (0.5, 1.0), (0.2, 1.0)):
        wq = w.with_(ar_rho=rho, drift_scale=drift)
        sub = layers[:2]
        paths = []
        for l in range(len(sub)):
            qs = W.QueryStream(wq, l, device)
            paths.append([qs.next() for _ in range(total)])
        for L in sub:
            L.slot_table.fill_(-1)
            L.last_used.fill_(-1)
            L.sel.fill_(-1)
        pipe = DecodePipeline(d, sub, ctx, 1.0 / math.sqrt(w.head_dim), device, exact="measure", steps_cap=total)
        pipe.build_summaries()
        pipe.prime([p[0] for p in paths])
        for t in range(1, total):
            pipe.step(t, [p[t] for p in paths])
        pipe.wait_all()
        c = pipe.prediction_counts()[:, :, fill:total - 1].double().mean(dim=(0, 2, 3, 4)) / float(w.budget_blocks)
        sweep.append({"ar_rho": rho, "drift_scale": drift, "lookahead_agreement": c[0].item(),
                      "previous_token_agreement": c[1].item(), "resident_coverage": c[2].item()})
        del pipe
    err = lsk.read_device_error(clear=True)
    line = {
        "metric": "top-K prediction agreement and corrective fetch (synthetic analog of OasisKV Figs. 4 and 6)",
        "workload": f"llama8b_32k_lead: {nl} Llama-3.1-8B-shaped layers at 32K, batch {w.batch}, budget "
                    f"{w.budget_blocks} blocks, cap {w.fetch_cap}, 1+{w.n_drafts} queries; draft j of step t "
                    f"is drawn around the query mean of step t+j (AR(1) rho {w.ar_rho})",
        "steps": args.steps, "warmup_steps": fill, "layers": nl,
        "definitions": {"lookahead_agreement": "|lookahead top-K of step t-1 & exact top-K of step t| / K",
                        "previous_token_agreement": "|exact top-K of step t-1 & exact top-K of step t| / K",
                        "resident_coverage": "|resident blocks before step t & exact top-K of step t| / K",
                        "exact top-K": "top-K under the same min/max bound with the verification query alone"},
        "runs": out, "query_drift_sweep": sweep, "device_error_word": err,
    }
    print(json.dumps(line), flush=True)


def run_ablation(args, device):
    """Fetch-ratio x victim-order sweep over the 32K Llama layers.  Every
    setting starts from a pool primed with the full top-K (uncapped), runs
    warm-up steps at its cap, then times --steps decode steps without the
    exact-set stage; a second, untimed pass over the same steps measures the
    coverage of the exact set (the residency decisions do not depend on it)."""
    w = W.WORKLOADS["llama8b_32k"]
    K = w.budget_blocks
    d_full = lsk.dims_for(w.with_(fetch_cap=K))
    nl = args.layers
    warm = 8
    total = 1 + warm + args.steps
    layers, qpaths = [], []
    for l in range(nl):
        host = torch.empty((w.batch, w.n_kv_heads, w.max_blocks, 2, w.block_tokens, w.head_dim),
                           dtype=torch.bfloat16, pin_memory=True)
        W.make_host_kv(w, layer=l, device=device, out=host)
        layers.append(LayerState(d_full, host, device))       # fetch lists sized for any cap <= K
        qs = W.QueryStream(w, l, device)
        qpaths.append([qs.next() for _ in range(total)])
    torch.cuda.synchronize()
    ctx = W.initial_ctx_len(w, device)
    scale = 1.0 / math.sqrt(w.head_dim)
    cover = torch.zeros((w.batch, w.n_kv_heads), dtype=torch.int32, device=device)
    rows = []
    # the first setting runs once untimed first, so no row pays for the GPU's clock ramp
    settings = [(0.10, "lru", False)] + [(r, v, True) for r in (0.01, 0.02, 0.05, 0.10, 0.20, 1.0)
                                         for v in ("lru", "score")]
    for ratio, victims, keep in settings:
        cap = max(1, round(ratio * K))
        d = lsk.dims_for(w.with_(fetch_cap=cap))
        res = {"fetch_ratio": ratio, "cap": cap, "victims": victims}
        for exact in ((None, "measure") if keep else (None,)):
            for L in layers:
                L.slot_table.fill_(-1)
                L.last_used.fill_(-1)
            primer = DecodePipeline(d_full, layers, ctx, scale, device, victims=victims)
            primer.build_summaries()
            primer.prime([p[0] for p in qpaths])
            primer.wait_all()
            torch.cuda.synchronize()
            del primer
            pipe = DecodePipeline(d, layers, ctx, scale, device, exact=exact, steps_cap=total, victims=victims)
            for t in range(1, 1 + warm):
                pipe.step(t, [p[t] for p in qpaths])
            pipe.wait_all()
            torch.cuda.synchronize()
            hist = fetch_history(args.steps, layers, device)
            resident_sel = torch.zeros((), dtype=torch.int64, device=device)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(pipe.main)
            for t in range(1 + warm, total):
                pipe.step(t, [p[t] for p in qpaths])
                if exact is None:
                    record_fetches(hist, t - 1 - warm, layers)
            pipe.wait_all()
            e1.record(pipe.main)
            torch.cuda.synchronize()
            if exact is None:
                ms = e0.elapsed_time(e1)
                nfetch = hist.sum().item() / (nl * args.steps)        # blocks per layer-step
                for L in layers:                                       # final plan's fetches landed
                    lsk.block_overlap(d, L.slot_table, L.sel, cover)
                    resident_sel += cover.sum()
                torch.cuda.synchronize()
                res.update({"layer_steps_per_s": nl * args.steps / (ms * 1e-3),
                            "fetch_mib_per_layer_step": nfetch * w.block_bytes / 2 ** 20,
                            "h2d_gbs": nfetch * w.block_bytes * nl * args.steps / (ms * 1e-3) / 1e9,
                            "selection_resident_after_fetch":
                                resident_sel.item() / (nl * w.batch * w.n_kv_heads * K)})
            else:
                c = pipe.prediction_counts()[:, 2, warm:total - 1].double()
                res["exact_coverage"] = c.mean().item() / K
            del pipe
        if keep:
            rows.append(res)
    line = {
        "metric": "fetch-cap and victim-order ablation (synthetic analog of OasisKV Table 2)",
        "workload": f"llama8b_32k: {nl} Llama-3.1-8B-shaped layers at 32K, batch {w.batch}, budget {K} blocks, "
                    f"1+{w.n_drafts} queries, AR(1)-drifting queries",
        "steps": args.steps, "warmup_steps": warm,
        "definitions": {"cap": "max(1, round(fetch_ratio * K)) blocks per (sequence, KV head) per step",
                        "exact_coverage": "|resident before step t & exact top-K of the true query| / K",
                        "selection_resident_after_fetch": "|resident after the last fetch & last selection| / K",
                        "victims": "lru = least recently used stale slot; score = lowest current lookahead score"},
        "rows": rows, "device_error_word": lsk.read_device_error(clear=True),
    }
    print(json.dumps(line), flush=True)


def run_longctx(args, device):
    """Budget x cap sweep of the 128K layer; each setting primed with the full
    top-K, warmed up, and timed over --steps decode steps (128 by default: two
    hops of the planted blocks), with isolated kernel times for the overlap."""
    base = W.WORKLOADS["longctx_128k"]
    nl = min(args.layers, 4)
    warm, steps = 8, args.steps
    total = 1 + warm + steps
    hosts, qpaths = [], []
    for l in range(nl):
        h = torch.empty((base.batch, base.n_kv_heads, base.max_blocks, 2, base.block_tokens, base.head_dim),
                        dtype=torch.bfloat16, pin_memory=True)
        W.make_host_kv(base, layer=l, device=device, out=h)
        hosts.append(h)
        qs = W.QueryStream(base, l, device)
        qpaths.append([qs.next() for _ in range(total)])
    torch.cuda.synchronize()
    h2d = measure_h2d_peak(device)
    ctx = W.initial_ctx_len(base, device)
    scale = 1.0 / math.sqrt(base.head_dim)
    rows = []
    for K in (128, 256):
        d_full = lsk.dims_for(base.with_(budget_blocks=K, fetch_cap=K))
        layers = [LayerState(d_full, hosts[l], device) for l in range(nl)]     # fetch lists fit any cap
        built = False
        for cap in (4, 8, 16, 32):
            w = base.with_(budget_blocks=K, fetch_cap=cap)
            d = lsk.dims_for(w)
            for L in layers:
                L.slot_table.fill_(-1)
                L.last_used.fill_(-1)
            primer = DecodePipeline(d_full, layers, ctx, scale, device)
            if not built:
                primer.build_summaries()
                built = True
            primer.prime([p[0] for p in qpaths])
            primer.wait_all()
            torch.cuda.synchronize()
            del primer
            pipe = DecodePipeline(d, layers, ctx, scale, device)
            for t in range(1, 1 + warm):
                pipe.step(t, [p[t] for p in qpaths])
            pipe.wait_all()
            torch.cuda.synchronize()
            hist = fetch_history(steps, layers, device)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(pipe.main)
            for t in range(1 + warm, total):
                pipe.step(t, [p[t] for p in qpaths])
                record_fetches(hist, t - 1 - warm, layers)
            pipe.wait_all()
            e1.record(pipe.main)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            per_ls = ms / (nl * steps)
            fetched = hist.sum()
            gbs = fetched.item() * w.block_bytes / (ms * 1e-3) / 1e9
            iso = isolated_kernel_ms({"pipe": pipe, "layers": layers, "dims": d, "qrings": [[qpaths[0][total - 1]]]},
                                     reps=5)
            iso.pop("_prefetch_blocks")
            rows.append({"budget_blocks": K, "cap": cap, "layer_steps_per_s": 1.0 / (per_ls * 1e-3),
                         "fetch_mib_per_layer_step": fetched.item() / (nl * steps) * w.block_bytes / 2 ** 20,
                         "h2d_gbs": gbs, "h2d_frac": gbs / h2d["peak_gbs"],
                         "overlap_efficiency": overlap_efficiency(iso, per_ls)["value"],
                         "compute_ms": overlap_efficiency(iso, per_ls)["compute_ms"],
                         "isolated_ms": {k: iso[k] for k in ("sparse_attn", "score_select_plan", "prefetch")}})
            del pipe
        del layers
        torch.cuda.empty_cache()
    line = {
        "metric": "128K long-context stress: budget x cap sweep (layer-steps/s, H2D vs PCIe roof, overlap efficiency)",
        "workload": f"longctx_128k: {nl} layers, batch 8, 32/8 heads, 131,072 tokens (8,192 blocks per head), "
                    f"Student-t(3) keys, 4 groups of 6 planted blocks hopping every 64 steps, 1+4 queries",
        "steps": steps, "warmup_steps": warm, "h2d_peak": h2d, "rows": rows,
        "device_error_word": lsk.read_device_error(clear=True),
    }
    print(json.dumps(line), flush=True)


def run_reasoning(args, device):
    """Long-output reasoning decode: 36 layers shaped like Qwen3-8B (batch 64,
    32/8 heads, budget 128 blocks, cap 8, 1+4 queries), one new token per
    sequence appended every step (host KV, summaries and the resident slot of
    its block updated in place).  The context is measured in four windows
    that start at 1K (the whole context fits the budget), 4K, 8K and just
    below 17K tokens: each window resets the pool, rebuilds the summaries of
    its starting context, primes, fills the pool over warm-up steps and times
    --steps (at most 32) decode steps.  Host KV: layers share the pinned KV of
    layer l mod L (L distinct layers, 4.6 GB each); the rows appended at a
    step are drawn per distinct layer, so layers that share host KV append
    identical rows and every layer's summaries and pool stay consistent with
    it."""
    base = W.WORKLOADS["qwen8b_reasoning"]
    nl = args.layers if args.layers_given else base.layers
    steps = min(args.steps, 32)
    warm = base.budget_blocks // max(1, base.fetch_cap) + 2
    total = 1 + warm + steps
    ring = 16
    cap_tokens = base.max_blocks * base.block_tokens                   # 17,408
    starts = [1024, 4096, 8192, cap_tokens - total - 8]
    try:
        distinct = host_kv_layers(base, nl, 1)
    except Exception:
        distinct = nl
    distinct = max(1, min(distinct, args.host_kv_layers or 4))
    d = lsk.dims_for(base)
    hosts = []
    for l in range(distinct):
        h = torch.empty((base.batch, base.n_kv_heads, base.max_blocks, 2, base.block_tokens, base.head_dim),
                        dtype=torch.bfloat16, pin_memory=True)
        W.make_host_kv(base, layer=l, device=device, out=h)
        hosts.append(h)
    layers = [LayerState(d, hosts[l % distinct], device) for l in range(nl)]
    qrings = []
    for l in range(nl):
        qs = W.QueryStream(base, l, device)
        qrings.append([qs.next() for _ in range(ring)])
    torch.cuda.synchronize()
    h2d = measure_h2d_peak(device)
    scale = 1.0 / math.sqrt(base.head_dim)
    rows = []
    for c0 in starts:
        # rows appended at decode steps 1 .. total-1, per distinct host layer
        apps = [[W.append_rows(base, l, c0 + t, device) for l in range(distinct)] for t in range(total)]
        for L in layers:
            L.slot_table.fill_(-1)
            L.last_used.fill_(-1)
        ctx = torch.full((base.batch,), c0, dtype=torch.int32, device=device)
        pipe = DecodePipeline(d, layers, ctx, scale, device)
        pipe.build_summaries()

        def qs_at(t):
            return [r[ring_index(t, ring)] for r in qrings]

        def app_at(t):
            return [apps[t][l % distinct] for l in range(nl)]

        pipe.prime(qs_at(0))
        for t in range(1, 1 + warm):
            pipe.step(t, qs_at(t), appended=app_at(t))
        pipe.wait_all()
        torch.cuda.synchronize()
        hist = fetch_history(steps, layers, device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(pipe.main)
        h0 = time.perf_counter()
        for t in range(1 + warm, total):
            pipe.step(t, qs_at(t), appended=app_at(t))
            record_fetches(hist, t - 1 - warm, layers)
        pipe.wait_all()
        e1.record(pipe.main)
        host_ms = (time.perf_counter() - h0) * 1e3
        torch.cuda.synchronize()
        fetched = hist.sum()
        ms = e0.elapsed_time(e1)
        ctx_end = int(pipe.ctx_len[0].item())
        per_ls = ms / (nl * steps)
        fetched_ls = fetched.item() / (nl * steps)
        gbs = fetched_ls * base.block_bytes / (per_ls * 1e-3) / 1e9
        w_now = base.with_(context=ctx_end)
        iso = isolated_kernel_ms({"pipe": pipe, "layers": layers, "dims": d, "qrings": [[qs_at(total - 1)[0]]]},
                                 reps=5)
        iso.pop("_prefetch_blocks")
        ab = algorithmic_bytes(w_now, fetched_ls)
        attn_gbs = ab["sparse_attn"] / (iso["sparse_attn"] * 1e-3) / 1e9
        rows.append({
            "context_start": c0, "context_end": ctx_end,
            "layer_steps_per_s": 1.0 / (per_ls * 1e-3), "tokens_per_s": 1.0 / (per_ls * 1e-3) / nl * base.batch,
            "fetched_blocks_per_layer_step": fetched_ls, "h2d_gbs": gbs, "h2d_frac": gbs / h2d["peak_gbs"],
            "overlap_efficiency": overlap_efficiency(iso, per_ls)["value"],
            "compute_ms": overlap_efficiency(iso, per_ls)["compute_ms"],
            "attention_hbm_gbs": attn_gbs, "host_enqueue_ms_per_step": host_ms / steps,
            "isolated_ms": {k: iso[k] for k in ("sparse_attn", "score_select_plan", "prefetch")}})
        del pipe
    line = {
        "metric": "long-output reasoning decode with appends: layer-steps/s, tokens/s, H2D vs PCIe roof, "
                  "overlap efficiency, per context window",
        "workload": f"qwen8b_reasoning: {nl} Qwen3-8B-shaped layers, batch 64, 32/8 heads, budget "
                    f"{base.budget_blocks} blocks, cap {base.fetch_cap}, 1+4 queries, one appended token per "
                    f"sequence per step; host KV of {distinct} distinct layers (l -> l mod {distinct})",
        "steps_per_window": steps, "warmup_steps": warm, "h2d_peak": h2d, "windows": rows,
        "gpu_launches_per_layer_step": launches_per_layer_step(base) + 1,     # + the append
        "device_error_word": lsk.read_device_error(clear=True),
    }
    print(json.dumps(line), flush=True)


def run_deep(args, device):
    """Eager vs graph-replayed decode steps of a 64-layer stack."""
    base = W.WORKLOADS["qwen32b_32k"]
    nl, distinct, ring = 64, 8, 16
    steps = min(args.steps, 48)
    rows = []
    for batch in (16, 2):
        w = base.with_(batch=batch)
        d = lsk.dims_for(w)
        hosts = []
        for l in range(distinct):
            h = torch.empty((w.batch, w.n_kv_heads, w.max_blocks, 2, w.block_tokens, w.head_dim),
                            dtype=torch.bfloat16, pin_memory=True)
            W.make_host_kv(w, layer=l, device=device, out=h)
            hosts.append(h)
        layers = [LayerState(d, hosts[l % distinct], device) for l in range(nl)]
        # queries of all layers for one step in one tensor, so a step costs one copy
        streams = [W.QueryStream(w, l, device) for l in range(nl)]
        qring = [torch.stack([qs.next() for qs in streams]) for _ in range(ring)]     # [ring][layers, B, Qn, Hq, D]
        q_all = torch.empty_like(qring[0])
        q_static = list(q_all)
        # the configuration's seeded residency loss, one mask per layer and step (ring like the queries)
        mring = [torch.stack([W.eviction_mask(w, l, r, device) for l in range(nl)]).to(torch.uint8)
                 for r in range(ring)]
        m_all = torch.empty_like(mring[0])
        m_static = list(m_all)
        ctx = W.initial_ctx_len(w, device)
        torch.cuda.synchronize()
        built = False
        for mode in ("eager", "graph"):
            for L in layers:
                L.slot_table.fill_(-1)
                L.last_used.fill_(-1)
            pipe = DecodePipeline(d, layers, ctx, 1.0 / math.sqrt(w.head_dim), device, device_step=(mode == "graph"))
            with torch.cuda.stream(pipe.main):
                if not built:
                    pipe.build_summaries()
                    built = True
                pipe.prime(list(qring[0]))
            t = 1

            def load_queries(t):
                with torch.cuda.stream(pipe.main):
                    q_all.copy_(qring[ring_index(t, ring)], non_blocking=True)
                    m_all.copy_(mring[ring_index(t, ring)], non_blocking=True)

            for _ in range(4):                         # warm-up, eager in both modes
                load_queries(t)
                with torch.cuda.stream(pipe.main):
                    pipe.step(t, q_static, evict=m_static)
                t += 1
            with torch.cuda.stream(pipe.main):
                pipe.wait_all()
            torch.cuda.synchronize()
            if mode == "graph":
                pipe.capture(q_static, evict_static=m_static)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            h0 = time.perf_counter()
            e0.record(pipe.main)
            for _ in range(steps):
                load_queries(t)
                if mode == "graph":
                    pipe.replay()
                else:
                    with torch.cuda.stream(pipe.main):
                        pipe.step(t, q_static, evict=m_static)
                t += 1
            with torch.cuda.stream(pipe.main):
                pipe.wait_all()
            e1.record(pipe.main)
            host_ms = (time.perf_counter() - h0) * 1e3
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            rows.append({"batch": batch, "mode": mode, "layer_steps_per_s": nl * steps / (ms * 1e-3),
                         "ms_per_step": ms / steps, "host_enqueue_ms_per_step": host_ms / steps,
                         "gpu_launches_per_step": 1 if mode == "graph" else None})
            del pipe
        del layers, hosts, qring, q_all, q_static, mring, m_all, m_static
        torch.cuda.empty_cache()
    line = {
        "metric": "decode step of a 64-layer stack: eager stream pipeline vs one CUDA graph replay per step",
        "workload": f"qwen32b_32k shape: {nl} layers (host KV of 8 distinct layers, l -> l mod 8), 64/8 heads, "
                    f"32K context, budget 128 blocks, cap 16, 1+7 queries; batch 16 and 2; "
                    f"seeded 10 % residency loss per step; every step copies all layers' queries and loss masks "
                    f"into fixed buffers (one copy each) in both modes",
        "steps": steps, "rows": rows, "device_error_word": lsk.read_device_error(clear=True),
    }
    print(json.dumps(line), flush=True)


def run_gpu(args, rank, world, device):
    w = rank_workload(rank, args.workload)
    nl = args.layers
    try:
        host_layers = host_kv_layers(w, nl, int(os.environ.get("LOCAL_WORLD_SIZE", world)))
    except Exception:                                   # no estimate: one host KV per layer, as asked
        host_layers = nl
    # the 64-layer stack's 128 GiB of host KV would pin most of a GPU node's
    # memory: by default 16 distinct layers (32 GiB) are pinned and shared
    cap = args.host_kv_layers or BENCH_WORKLOADS[args.workload]["host_kv_cap"]
    if cap:
        host_layers = min(host_layers, cap)
    st = build_workload_state(w, args.warmup + args.steps, device, n_queries=args.query_ring,
                              layers=nl, host_layers=host_layers)
    st["host_layers"] = host_layers
    d, layers, pipe, qrings, mrings = st["dims"], st["layers"], st["pipe"], st["qrings"], st["mrings"]
    nq = len(qrings[0])
    timer = KernelTimer(args.steps * nl)
    pipe.timer = timer
    main = pipe.main
    fetch_hist = fetch_history(args.steps, layers)

    def qs_at(t):
        i = ring_index(t, nq)
        return [r[i] for r in qrings]

    def ms_at(t):                                       # the step's residency-loss masks, or None
        if mrings is None:
            return None
        i = ring_index(t, nq)
        return [r[i] for r in mrings]

    pipe.prime(qs_at(0))
    t = 1
    for _ in range(args.warmup):
        pipe.step(t, qs_at(t), evict=ms_at(t))
        t += 1
    pipe.wait_all()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    timer.on = True
    with ClockSampler(torch.cuda.current_device()) as clk:
        ev0.record(main)
        h0 = time.perf_counter()
        for i in range(args.steps):
            pipe.step(t, qs_at(t), evict=ms_at(t))
            record_fetches(fetch_hist, i, layers)
            t += 1
        pipe.wait_all()
        ev1.record(main)
        host_ms = (time.perf_counter() - h0) * 1e3
        torch.cuda.synchronize()
    timer.on = False
    ms = ev0.elapsed_time(ev1)
    if world > 1:
        torch.distributed.barrier()
    ms = max_over_ranks(ms)

    # host cost of a step: a few steps enqueued right after a synchronize, so the
    # launch queue has room and the host never waits on the device
    host_cost = []
    for _ in range(3):
        torch.cuda.synchronize()
        h0 = time.perf_counter()
        for _ in range(4):
            pipe.step(t, qs_at(t), evict=ms_at(t))
            t += 1
        host_cost.append((time.perf_counter() - h0) * 1e3 / 4)
    pipe.wait_all()
    torch.cuda.synchronize()

    # reuse of the selected set between consecutive steps (untimed)
    reuse = []
    prev = [L.sel.clone() for L in layers]
    for _ in range(8):
        pipe.step(t, qs_at(t), evict=ms_at(t))
        t += 1
        pipe.wait_all()
        for l, L in enumerate(layers):
            cur = L.sel.clone()
            same = (cur.unsqueeze(-1) == prev[l].unsqueeze(-2)) & (cur.unsqueeze(-1) >= 0)
            reuse.append(same.any(-1).sum().item() / max(1, (cur >= 0).sum().item()))
            prev[l] = cur
    torch.cuda.synchronize()

    # end-to-end through the API: every step copies each layer's queries in
    # from pinned host memory (input stream, one event per layer) and reads
    # each layer's outputs back once that layer is done (output stream); the
    # host waits for the last read-back before it starts the next step.  The
    # residency-loss masks stand for the memory system, not for a caller's
    # input, and stay on the device.
    e2e_steps = min(args.steps, 200)
    hq = [[q.cpu().pin_memory() for q in r[: min(nq, 32)]] for r in qrings]
    qdev = [torch.empty_like(r[0]) for r in qrings]
    hout = [torch.empty(L.out.shape, dtype=L.out.dtype, pin_memory=True) for L in layers]
    hlse = [torch.empty(L.lse.shape, dtype=L.lse.dtype, pin_memory=True) for L in layers]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    in_ev = [torch.cuda.Event() for _ in layers]
    out_ev = [torch.cuda.Event() for _ in layers]
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    s_in.wait_event(e0)
    for i in range(e2e_steps):
        j = ring_index(i, len(hq[0]))
        with torch.cuda.stream(s_in):
            for l in range(nl):
                qdev[l].copy_(hq[l][j], non_blocking=True)
                in_ev[l].record(s_in)
        pipe.step(t, qdev, evict=ms_at(t), inputs_ready=in_ev, layer_done=out_ev)
        t += 1
        with torch.cuda.stream(s_out):
            for l, L in enumerate(layers):
                s_out.wait_event(out_ev[l])
                hout[l].copy_(L.out, non_blocking=True)
                hlse[l].copy_(L.lse, non_blocking=True)
        s_out.synchronize()
    pipe.wait_all()
    e1.record(main)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    del hq, hout, hlse

    iso = isolated_kernel_ms(st)
    h2d = measure_h2d_peak(device) if rank == 0 else None
    err = lsk.read_device_error(clear=True)
    return {"w": w, "name": args.workload, "d": d, "ms": ms, "host_ms": host_ms, "host_cost_ms": min(host_cost),
            "timer": timer, "fetch_hist": fetch_hist, "reuse": reuse,
            "e2e_ms": e2e_ms, "e2e_steps": e2e_steps, "h2d": h2d, "clocks": clk.summary(), "dev_err": err,
            "layer": layers[0], "layers": layers, "queries": qrings[0],
            "masks": None if mrings is None else mrings[0], "iso": iso,
            "host_layers": st["host_layers"]}


def algorithmic_bytes(w, fetched_blocks_per_layer_step):
    """Bytes each kernel must move per launch (the whole batch, one layer)."""
    units = w.batch * w.n_kv_heads
    nv = math.ceil(w.context / w.block_tokens)
    q_bytes = w.batch * w.n_queries * w.n_q_heads * w.head_dim * 2
    out_bytes = w.batch * w.n_queries * w.n_q_heads * (w.head_dim + 1) * 4
    block = w.block_bytes
    return {
        # resident KV (every slot is occupied after warm-up) + queries + outputs
        "sparse_attn": units * w.budget_blocks * block + q_bytes + out_bytes,
        # min/max summaries of every valid block + draft queries + scores written and read + selection
        # plus the plan's slot table / recency read and written and its fetch lists
        "score_select_plan": (units * nv * 2 * w.head_dim * 2 + q_bytes + 2 * units * nv * 4
                              + units * w.budget_blocks * 8 + units * w.budget_blocks * 4 * 4
                              + units * w.fetch_cap * 8 + units * 4),
        "select_only": units * nv * 4 + units * w.budget_blocks * 8,
        # slot table + last-used read and written, selection read, fetch lists written
        "plan_fetch": units * w.budget_blocks * 4 * 5 + units * w.fetch_cap * 8 + units * 4,
        # fetched blocks: read over PCIe and written to HBM (counted once, as H2D bytes)
        "prefetch": fetched_blocks_per_layer_step * block,
        # a1 at admission: the K half of every valid block read over PCIe (the summaries it writes,
        # 1/8 of that, go to HBM and are not counted against the link)
        "build_summaries": units * nv * (block // 2),
    }


def overlap_efficiency(iso_ms, pipeline_ms_per_layer_step):
    """eta = (T_compute + T_fetch - T_pipeline) / min(T_compute, T_fetch) per
    layer-step: 1 when the gather hides completely behind (or hides) the
    compute, 0 when they run back to back.  T_fetch is the isolated gather;
    T_compute the compute path of a layer-step as the pipeline runs it on
    one stream: attention + (scores, top-K and plan in one launch), from
    isolated times.  T_pipeline is the measured per-layer-step time of the
    pipeline."""
    t_c = iso_ms["sparse_attn"] + iso_ms["score_select_plan"]
    t_f = iso_ms["prefetch"]
    return {"value": (t_c + t_f - pipeline_ms_per_layer_step) / min(t_c, t_f),
            "compute_ms": t_c, "fetch_ms": t_f, "pipeline_ms": pipeline_ms_per_layer_step}


def token_kv_intensity(w, fetched_blocks_per_layer_step):
    """OasisKV Figure 1: how many new tokens a decode pass yields for each
    KV-cache byte it moves, per memory tier (HBM, PCIe); one token per
    sequence per layer-step."""
    units = w.batch * w.n_kv_heads
    nv = math.ceil(w.context / w.block_tokens)
    hbm = units * w.budget_blocks * w.block_bytes + units * nv * 2 * w.head_dim * 2   # resident KV + summaries
    io = fetched_blocks_per_layer_step * w.block_bytes
    dense = units * nv * w.block_bytes
    mib = float(2 ** 20)
    return {"hbm_tokens_per_mib": w.batch / (hbm / mib), "pcie_tokens_per_mib": w.batch / (io / mib) if io else None,
            "dense_hbm_tokens_per_mib": w.batch / (dense / mib),
            "definition": "batch tokens per MiB of KV-cache bytes per layer-step: HBM = resident KV + block summaries "
                          "read; PCIe = fetched blocks; dense = the whole KV read by dense attention"}


def launches_per_layer_step(w) -> int:
    """Kernels of one layer-step: attention, scores + top-K + plan (one
    launch) and gather, plus the residency loss when the workload has one."""
    return 3 + (1 if w.evict_prob > 0 else 0)


def emit_gpu(args, res, world):
    w, timer = res["w"], res["timer"]
    nl = len(res["layers"])
    peaks, peak_src = load_peaks()
    layer_steps = args.steps * nl
    fetched = res["fetch_hist"].sum().item() / layer_steps            # blocks per layer-step (this rank)
    ab = algorithmic_bytes(w, fetched)
    h2d_peak = res["h2d"]["peak_gbs"] if res["h2d"] else None
    traffic = load_traffic(w.name)

    def roof(k, ms):
        gbs = ab[k] / (ms * 1e-3) / 1e9
        if k in ("prefetch", "build_summaries"):
            bound, peak, src = "h2d", h2d_peak, "measured in this run (best of 1 GiB pinned memcpy, zero-copy gather)"
        else:
            bound, peak, src = "hbm", peaks["hbm_gbs"], f"{peak_src} hbm_gbs (MEASURED_PEAKS)"
        return {"ms": ms, "bytes": ab[k], "achieved_gbs": gbs, "bound": bound, "peak_gbs": peak,
                "frac": (gbs / peak) if peak else None, "peak_source": src, "traffic": traffic.get(k)}

    kernels = {k: roof(k, timer.mean_ms(k)) for k in KERNELS if timer.mean_ms(k) is not None}
    iso = dict(res["iso"])
    iso_blocks = iso.pop("_prefetch_blocks")
    isolated = {k: roof(k, v) for k, v in iso.items()}
    isolated["prefetch"]["bytes"] = iso_blocks * w.block_bytes
    isolated["prefetch"]["achieved_gbs"] = iso_blocks * w.block_bytes / (iso["prefetch"] * 1e-3) / 1e9
    if h2d_peak:
        isolated["prefetch"]["frac"] = isolated["prefetch"]["achieved_gbs"] / h2d_peak
    dominant = max(kernels, key=lambda k: kernels[k]["ms"])
    kd = kernels[dominant]
    value = world * layer_steps / (res["ms"] * 1e-3)
    e2e_value = world * res["e2e_steps"] * nl / (res["e2e_ms"] * 1e-3)
    q_bytes = w.batch * w.n_queries * w.n_q_heads * w.head_dim * 2
    L = res["layer"]
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "layer-steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": res["ms"] / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": data_label(w),
        "config": headline_config(w, nl, world, res.get("name", WORKLOAD)),
        "roofline": {"kernel": dominant, "bound": kd["bound"], "achieved": kd["achieved_gbs"],
                     "peak": kd["peak_gbs"], "unit": "GB/s", "frac": kd["frac"], "traffic": kd["traffic"],
                     "peak_source": kd["peak_source"]},
        "kernels": kernels,
        "kernels_isolated": isolated,
        "tokens_per_s": value / nl * w.batch,
        "fetched_blocks_per_layer_step": fetched,
        "h2d_gbs_avg": ab["prefetch"] * layer_steps / (res["ms"] * 1e-3) / 1e9,
        "reuse": sum(res["reuse"]) / len(res["reuse"]),
        "overlap_efficiency": overlap_efficiency(iso, res["ms"] / layer_steps),
        "token_kv_intensity": token_kv_intensity(w, fetched),
        "h2d_peak": res["h2d"],
        "e2e": {"value": e2e_value, "unit": "layer-steps/s",
                "h2d_bytes_per_step": nl * (q_bytes + int(ab["prefetch"])),
                "d2h_bytes_per_step": nl * (L.out.numel() * 4 + L.lse.numel() * 4),
                "note": "per step: every layer's queries copied in from pinned host memory and its outputs read "
                        "back as soon as that layer is done, the host waiting for the last read-back before the "
                        "next step; h2d bytes include the zero-copy gather of fetched blocks"},
        "gpu_launches": launches_per_layer_step(w) * layer_steps,
        "host_kv_layers": res.get("host_layers", nl),   # distinct pinned host KV per rank (layer l -> l mod this)
        "cpus_bound": res.get("cpus_bound"),   # rank 0's CPUs local to its GPU (multi-rank runs), else null
        "host_enqueue_ms_per_step": res["host_ms"] / args.steps,
        "host_cost_ms_per_step": res["host_cost_ms"],
        "clocks": res["clocks"],
        "device_error_word": res["dev_err"],
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, res)
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------- oracle
def oracle_cfg(w) -> dict:
    """The workload fields the oracle's per-unit driver needs."""
    return {"context": w.context, "block_tokens": w.block_tokens, "budget_blocks": w.budget_blocks,
            "head_dim": w.head_dim, "fetch_cap": w.fetch_cap}


def cpu_baseline(w, res, n_units=6, fill_steps=8, timed_steps=24, par_fill=4, par_timed=8):
    """The oracle, as it stands, on this host's cores, on a sample of the
    benchmarked workload (the same KV and queries), in layer-steps/s of the
    whole batch: on one core (a few units one after another) and on all
    usable cores (one unit per core, all at once).  `value` is the all-cores
    figure when that run succeeds, else the one-core figure."""
    import numpy as np

    import oracle as O
    from oracle import decode_timing as T
    L = res["layer"]
    G = w.group
    total_units = w.batch * w.n_kv_heads
    qs_all = [O.bf16_bits_to_f64(W.bf16_bits(q)) for q in res["queries"][: fill_steps + timed_steps + 1]]
    ms_all = None
    if res.get("masks") is not None:                   # the same loss masks the GPU run used
        ms_all = [m.cpu().numpy().astype(bool) for m in res["masks"][: fill_steps + timed_steps + 1]]

    def unit(b, h, steps):
        masks = None if ms_all is None else [m[b:b + 1, h:h + 1] for m in ms_all[:steps]]
        return (W.bf16_bits(L.host_kv[b:b + 1, h:h + 1]), [q[b:b + 1, :, h * G:(h + 1) * G] for q in qs_all[:steps]],
                masks)

    rng = np.random.default_rng(0)
    picks = [(int(rng.integers(w.batch)), int(rng.integers(w.n_kv_heads))) for _ in range(n_units)]
    times = []
    for b, h in picks:
        bits, qs, masks = unit(b, h, fill_steps + timed_steps + 1)
        times += T.run_unit(oracle_cfg(w), bits, qs, fill_steps, timed_steps, masks=masks)
    one = 1.0 / (sum(times) / len(times) * total_units)
    single = {"value": one, "unit": "layer-steps/s", "cores": 1,
              "sample": f"{len(times)} unit-steps ({n_units} (sequence, KV head) units x {timed_steps} decode "
                        f"layer-steps after {fill_steps} untimed fill steps) one after another; per-unit mean "
                        f"scaled to the {total_units} units of the batch"}
    line = {"value": one, "unit": "layer-steps/s", "cores": 1, "kind": "oracle",
            "sample": single["sample"] + "; numpy fp64, BLAS 1 thread", "single_core": single,
            "nproc": os.cpu_count(), "usable_cores": T.usable_cores(), "cpu_model": T.cpu_model()}
    workers = max(1, min(T.usable_cores(), 64, total_units))          # one process (≈0.2 GB) per unit
    try:
        flat = [(b, h) for b in range(w.batch) for h in range(w.n_kv_heads)]
        order = rng.permutation(len(flat))[:workers]
        units = [unit(*flat[i], par_fill + par_timed + 1) for i in order]
        per_unit = T.run_units_parallel(oracle_cfg(w), units, par_fill, par_timed, workers, timeout_s=300.0)
        rate = sum(len(t) / sum(t) for t in per_unit)                 # unit-steps/s, all cores together
        line.update({"value": rate / total_units, "cores": workers,
                     "sample": f"{workers} (sequence, KV head) units, one per core, started together, each "
                               f"{par_timed} timed decode layer-steps after {par_fill} untimed fill steps; the "
                               f"sum of the units' step rates scaled to the {total_units} units of the batch; "
                               f"numpy fp64, BLAS 1 thread per process"})
    except Exception as e:                                            # one core stays the baseline
        line["all_cores_error"] = f"{type(e).__name__}: {e}"[:200]
    return line


def run_reference(args):
    """--impl reference: the CPU oracle on this host's cores, same workload,
    metric, unit and config as the GPU arm.  Each timed step is one decode
    layer-step (attention, residency loss, scores, top-K, plan, gather) of
    the whole batch at one layer: every (sequence, KV head) unit of the batch,
    spread over one process per usable core (at most 64), timed by the wall
    clock from the start of the step to the last process's reply.  Every
    layer of the stack has the same shape and work, so layer-steps/s is the
    number of timed layer-steps over their time, with no scaling; a step of
    this arm is one layer-step, and ms_per_step is its time.  --ref-units U
    (quick checks only) times the first U units and scales to the batch, and
    says so in its sample."""
    import oracle as O
    from oracle import decode_timing as T
    w = W.WORKLOADS[args.workload]
    total_units = w.batch * w.n_kv_heads
    n_units = total_units if not args.ref_units else max(1, min(args.ref_units, total_units))
    P = max(1, min(T.usable_cores(), 64, n_units))
    wu = w.with_(batch=-(-n_units // w.n_kv_heads))
    kv = W.make_host_kv(wu, 0, "cpu")
    qs = W.QueryStream(wu, 0, "cpu")
    ring_n = 16
    ring = [O.bf16_bits_to_f64(W.bf16_bits(qs.next())) for _ in range(ring_n)]   # walked in order, then again
    masks = None
    if w.evict_prob > 0:
        masks = [W.eviction_mask(wu, 0, i, "cpu").numpy() for i in range(ring_n)]
    G, fill = w.group, 4
    units = []
    for k in range(n_units):
        b, h = divmod(k, w.n_kv_heads)
        units.append((W.bf16_bits(kv[b:b + 1, h:h + 1]), [q[b:b + 1, :, h * G:(h + 1) * G] for q in ring],
                      None if masks is None else [m[b:b + 1, h:h + 1] for m in masks]))
    del kv
    loss = ", residency loss," if masks is not None else ""
    what = (f"decode layer-step (attention{loss} scores, top-K, plan, gather) of {n_units} (sequence, KV head) units "
            f"of {args.workload} at one layer; numpy fp64, BLAS 1 thread per process")
    scaled = n_units != total_units
    try:
        with T.UnitPool(oracle_cfg(wu), units, fill, timeout_s=1500.0, workers=P) as pool:
            for _ in range(args.warmup):
                pool.step()
            walls = [pool.step()[0] for _ in range(args.steps)]
        cores = P
        sample = (f"each step: one {what}, the units spread over {P} processes (one per core) and stepped "
                  f"together, wall clock from start to the last reply")
    except Exception as e:                                            # one core
        walls = []
        times = [T.run_unit(oracle_cfg(wu), *u[:2], fill + args.warmup, args.steps, masks=u[2])
                 for u in units[: max(1, min(4, n_units))]]
        per_step = [sum(t[i] for t in times) / len(times) for i in range(args.steps)]
        walls = [x * n_units for x in per_step]
        cores = 1
        sample = (f"each step: {len(times)} units' {what.split(' of ', 1)[0]} on one core, the mean scaled to "
                  f"{n_units} units (the all-cores run failed: {type(e).__name__})")
    ms = sum(walls) / len(walls) * 1e3 * (total_units / n_units)
    if scaled:
        sample += f"; scaled from {n_units} to the {total_units} units of the batch"
    value = 1e3 / ms
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value, "unit": "layer-steps/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "step_layers": 1, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": data_label(w),
        "config": headline_config(w, args.layers, args.gpus, args.workload),
        "cpu_baseline": {"value": value, "unit": "layer-steps/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "layer-steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1, help="GPUs (one rank each under torchrun; weak scaling)")
    ap.add_argument("--steps", type=int, default=50, help="timed decode steps (each runs every layer)")
    ap.add_argument("--warmup", type=int, default=10, help="untimed steps before them (at least 3)")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(BENCH_WORKLOADS),
                    help="benchmarked stack (default: the 64-layer Qwen3-32B-shaped one with residency loss)")
    ap.add_argument("--layers", type=int, default=None, help="pipelined attention layers per step "
                    "(default: the workload's, 64 or 8)")
    ap.add_argument("--host-kv-layers", type=int, default=0,
                    help="most distinct pinned host-KV layers (0: the workload's default cap, 16 for the "
                         "64-layer stack, within what the node's memory holds)")
    ap.add_argument("--query-ring", type=int, default=None,
                    help="pre-generated query steps, walked back and forth (default: the workload's)")
    ap.add_argument("--ref-units", type=int, default=0,
                    help="reference arm, quick checks only: time this many units and scale to the batch")
    ap.add_argument("--impl", default="oasis", choices=["oasis", "reference"],
                    help="reference: the CPU oracle on the host cores, same metric and config")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing in the GPU line")
    ap.add_argument("--prediction", action="store_true",
                    help="measure prediction agreement and the corrective fetch instead")
    ap.add_argument("--ablation", action="store_true",
                    help="fetch-cap x victim-order sweep (Table 2 analog) instead")
    ap.add_argument("--deep", action="store_true",
                    help="64-layer stack, eager vs CUDA-graph replay, instead")
    ap.add_argument("--longctx", action="store_true",
                    help="128K layer: budget x cap sweep with overlap efficiency, instead")
    ap.add_argument("--reasoning", action="store_true",
                    help="36-layer Qwen3-8B reasoning decode with appends, context windows 1K-17K, instead")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    spec = BENCH_WORKLOADS[args.workload]
    args.layers_given = args.layers is not None
    side_mode = args.prediction or args.ablation or args.deep or args.longctx or args.reasoning
    # the side modes run their own workloads; their stacks default to 8 layers
    args.layers = args.layers or (8 if side_mode else spec["layers"])
    args.query_ring = args.query_ring or spec["ring"]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    modes = [(args.prediction, run_prediction), (args.ablation, run_ablation), (args.deep, run_deep),
             (args.longctx, run_longctx), (args.reasoning, run_reasoning)]
    for on, fn in modes:
        if on:
            if rank == 0:
                fn(args, device)
            return
    bound = None
    if world > 1:
        import datetime
        bound = bind_near_gpu(device)                    # before any pinned host memory is allocated
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    try:
        res = run_gpu(args, rank, world, device)
        res["cpus_bound"] = bound
        if rank == 0:
            emit_gpu(args, res, world)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
