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
    iso = {"sparse_attn": 0.04, "score_select": 0.05, "plan_fetch": 0.01, "prefetch": 0.25}
    t_c, t_f = 0.06, 0.25                 # max(attention, scores + top-K) + plan
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
