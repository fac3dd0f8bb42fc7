"""Edge cases and maximum sizes on the GPU against the oracle: a sequence
with no context, the largest block count and budget the library accepts,
and gathers over more (sequence, KV head) units than one pass of the gather
kernel's prefix scan covers, with sparse fetch counts under a large cap."""

import math

import numpy as np
import pytest
import torch

import lookahead_sparse_kv_b200 as lsk
import oracle as O
from lookahead_sparse_kv_b200 import workloads as W
from tests.gpu_util import assert_attention_close, assert_selection_matches, f64, kv_split, np_i32, random_kv

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from lookahead_sparse_kv_b200 import build
    build.build()
    lsk.lib()
    yield
    assert lsk.read_device_error(clear=True) == 0


def test_sequence_with_no_context_runs_every_step():
    """ctx_len = 0: no valid block, an empty selection, nothing fetched, and
    attention gives 0 with lse -inf; the other sequence is unaffected."""
    B, Hq, Hkv, N, K, Qn, C = 2, 8, 2, 64, 16, 5, 4
    d = lsk.make_dims(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, max_blocks=N, budget_blocks=K, n_queries=Qn,
                      fetch_cap=C)
    g = torch.Generator()
    g.manual_seed(3)
    host = random_kv(B, Hkv, N, g).pin_memory()
    keys, vals = kv_split(host)
    ctx = torch.tensor([0, 700], dtype=torch.int32)
    cnp = ctx.numpy()
    q = torch.randn(B, Qn, Hq, 128, generator=g).to(torch.bfloat16)
    kmin = torch.zeros((B, Hkv, N, 128), dtype=torch.bfloat16, device=DEV)
    kmax = torch.zeros_like(kmin)
    ws = torch.zeros(lsk.workspace_bytes(d), dtype=torch.uint8, device=DEV)
    sel = torch.full((B, Hkv, K), -7, dtype=torch.int32, device=DEV)
    st = torch.full((B, Hkv, K), -1, dtype=torch.int32, device=DEV)
    lu = torch.full_like(st, -1)
    fs = torch.full((B, Hkv, C), -9, dtype=torch.int32, device=DEV)
    fb = torch.full_like(fs, -9)
    nf = torch.full((B, Hkv), -9, dtype=torch.int32, device=DEV)
    pool = torch.zeros((B, Hkv, K, 2, 16, 128), dtype=torch.bfloat16, device=DEV)
    out = torch.full((B, Qn, Hq, 128), 7.0, device=DEV)
    lse = torch.full((B, Qn, Hq), 7.0, device=DEV)
    ctx_d, qd = ctx.to(DEV), q.to(DEV)
    lsk.build_summaries(d, host, ctx_d, kmin, kmax)
    lsk.score_select(d, qd, kmin, kmax, ctx_d, sel, None, ws)
    lsk.plan_fetch(d, sel, st, lu, 0, fs, fb, nf)
    lsk.prefetch(d, host, fs, fb, nf, pool)
    lsk.sparse_attn(d, qd, pool, st, ctx_d, 1 / math.sqrt(128), out, lse, ws)
    torch.cuda.synchronize()
    omin, omax = O.block_summaries(keys, cnp)
    sc = O.lookahead_scores(f64(q), omin, omax, cnp, 16)
    ref_sel, _ = O.select_topk(sc, cnp, K, 16)
    g_sel = np_i32(sel)
    assert (g_sel[0] == -1).all() and (ref_sel[0] == -1).all()
    assert_selection_matches(g_sel[1:], ref_sel[1:], sc[1:], cnp[1:], K)
    plan = O.plan_fetch(g_sel, np.full((B, Hkv, K), -1, np.int32), np.full((B, Hkv, K), -1, np.int32), 0, C)
    np.testing.assert_array_equal(np_i32(st), plan["slot_table"])
    np.testing.assert_array_equal(np_i32(nf), plan["n_fetch"])
    assert (np_i32(nf)[0] == 0).all()
    stp = plan["slot_table"]
    pk = np.zeros((B, Hkv, K, 16, 128))
    pv = np.zeros_like(pk)
    for b in range(B):
        for h in range(Hkv):
            for s in range(K):
                if stp[b, h, s] >= 0:
                    pk[b, h, s], pv[b, h, s] = keys[b, h, stp[b, h, s]], vals[b, h, stp[b, h, s]]
    o_ref, lse_ref = O.sparse_attention(f64(q), pk, pv, stp, cnp, 1 / math.sqrt(128))
    assert_attention_close(out, lse, o_ref, lse_ref)
    assert (out[0] == 0).all() and torch.isinf(lse[0]).all() and (lse[0] < 0).all()


def test_select_at_the_largest_block_count_and_budget():
    """N = 32768 blocks and K = 1024 slots (the library's limits), bit-exact."""
    B, H, N, K = 1, 2, 32768, 1024
    d = lsk.make_dims(batch=B, n_q_heads=H, n_kv_heads=H, max_blocks=N, budget_blocks=K, n_queries=1,
                      fetch_cap=1)
    g = torch.Generator()
    g.manual_seed(11)
    s = torch.randint(-2000, 2000, (B, H, N), generator=g).float() * 0.5      # ties at the boundary
    ctx = torch.tensor([N * 16 - 5], dtype=torch.int32)
    sel = torch.empty((B, H, K), dtype=torch.int32, device=DEV)
    sel_s = torch.empty((B, H, K), device=DEV)
    lsk.select_topk(d, s.to(DEV), ctx.to(DEV), sel, sel_s)
    torch.cuda.synchronize()
    ref, ref_s = O.select_topk(s.numpy(), ctx.numpy(), K, 16)
    np.testing.assert_array_equal(np_i32(sel), ref)
    np.testing.assert_array_equal(sel_s.cpu().numpy(), ref_s)


def test_attention_at_the_largest_budget():
    """K = 1024 resident slots per head (the budget limit), 20 query rows."""
    B, Hq, Hkv, K, N, Qn = 1, 8, 2, 1024, 1100, 5
    d = lsk.make_dims(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, max_blocks=N, budget_blocks=K, n_queries=Qn,
                      fetch_cap=4)
    g = torch.Generator()
    g.manual_seed(12)
    kv = random_kv(B, Hkv, N, g)
    keys, vals = kv_split(kv)
    q = torch.randn(B, Qn, Hq, 128, generator=g).to(torch.bfloat16)
    ctx = torch.tensor([N * 16 - 3], dtype=torch.int32)
    rng = np.random.default_rng(12)
    st = np.stack([rng.permutation(N)[:K] for _ in range(Hkv)])[None].astype(np.int32)
    st[0, 1, ::7] = -1
    pool = torch.zeros((B, Hkv, K, 2, 16, 128), dtype=torch.bfloat16)
    for h in range(Hkv):
        for s_ in range(K):
            if st[0, h, s_] >= 0:
                pool[0, h, s_] = kv[0, h, st[0, h, s_]]
    out = torch.empty((B, Qn, Hq, 128), device=DEV)
    lse = torch.empty((B, Qn, Hq), device=DEV)
    ws = torch.zeros(lsk.workspace_bytes(d), dtype=torch.uint8, device=DEV)
    lsk.sparse_attn(d, q.to(DEV), pool.to(DEV), torch.from_numpy(st).to(DEV), ctx.to(DEV), 1 / math.sqrt(128),
                    out, lse, ws)
    torch.cuda.synchronize()
    pk, pv = kv_split(pool)
    o_ref, lse_ref = O.sparse_attention(f64(q), pk, pv, st, ctx.numpy(), 1 / math.sqrt(128))
    assert_attention_close(out, lse, o_ref, lse_ref)


@pytest.mark.parametrize("B,H,C,K,seed", [(50, 26, 3, 4, 0),        # 1300 units: two prefix passes
                                          (4, 8, 64, 64, 1),         # uncapped, sparse counts
                                          (1, 1, 1, 1, 2)])          # one unit, one entry
def test_gather_many_units_and_sparse_counts(B, H, C, K, seed):
    N = 6 if B * H > 1000 else 70
    d = lsk.make_dims(batch=B, n_q_heads=H, n_kv_heads=H, max_blocks=N, budget_blocks=K, n_queries=1,
                      fetch_cap=C)
    g = torch.Generator()
    g.manual_seed(seed)
    kv = torch.randint(-30000, 30000, (B, H, N, 2, 16, 128), dtype=torch.int16, generator=g)
    kv = kv.view(torch.bfloat16).pin_memory()
    rng = np.random.default_rng(seed)
    fs = np.full((B, H, C), -1, dtype=np.int32)
    fb = np.full((B, H, C), -1, dtype=np.int32)
    nf = rng.integers(0, min(C, 3) + 1, size=(B, H)).astype(np.int32)   # at most 3 real entries per unit
    nf.flat[0] = min(C, K)
    for b in range(B):
        for h in range(H):
            n = nf[b, h]
            fs[b, h, :n] = rng.permutation(K)[:n]
            fb[b, h, :n] = rng.permutation(N)[:n]
    pool = torch.randint(-30000, 30000, (B, H, K, 2, 16, 128), dtype=torch.int16, generator=g).view(torch.bfloat16)
    pool_d = pool.to(DEV)
    lsk.prefetch(d, kv, torch.from_numpy(fs).to(DEV), torch.from_numpy(fb).to(DEV), torch.from_numpy(nf).to(DEV),
                 pool_d)
    torch.cuda.synchronize()
    ref = O.prefetch(W.bf16_bits(kv), W.bf16_bits(pool), fs, fb, nf)
    np.testing.assert_array_equal(W.bf16_bits(pool_d), ref)
