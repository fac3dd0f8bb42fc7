"""CUDA path vs the CPU oracle, stage by stage, through the C ABI.

Each GPU stage is fed the same bytes as the oracle (usually the GPU's own
output of the previous stage) and compared element by element: summaries,
selections (given identical scores), plans and copied bytes bit-exactly;
scores within 1e-5 relative; selections from scratch up to the tie rule;
attention within abs 2e-3 / rel 1e-2."""

import math

import numpy as np
import pytest
import torch

import lookahead_sparse_kv_b200 as lsk
import oracle as O
from lookahead_sparse_kv_b200 import workloads as W
from tests.gpu_util import (SCORE_REL, assert_attention_close, assert_selection_matches, f64, kv_split,
                            np_i32, random_kv)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from lookahead_sparse_kv_b200 import build
    build.build()
    lsk.lib()
    torch.cuda.init()
    yield
    assert lsk.read_device_error(clear=True) == 0


def _dims(B, Hq, Hkv, N, K, Qn, C):
    return lsk.make_dims(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, max_blocks=N, budget_blocks=K,
                         n_queries=Qn, fetch_cap=C)


def _gen(seed):
    g = torch.Generator()
    g.manual_seed(seed)
    return g


# ------------------------------------------------------------- summaries
@pytest.mark.parametrize("host", [False, True])
def test_build_summaries(host):
    B, H, N = 3, 2, 37
    d = _dims(B, 8, H, N, 8, 5, 4)
    kv = random_kv(B, H, N, _gen(1))
    ctx = torch.tensor([N * 16, 16 * 20 + 7, 5], dtype=torch.int32)
    src = kv.pin_memory() if host else kv.to(DEV)
    kmin = torch.full((B, H, N, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    kmax = kmin.clone()
    lsk.build_summaries(d, src, ctx.to(DEV), kmin, kmax)
    torch.cuda.synchronize()
    keys, _ = kv_split(kv)
    omin, omax = O.block_summaries(keys, ctx.numpy())
    gmin, gmax = f64(kmin), f64(kmax)
    valid = ~np.isnan(omin)
    np.testing.assert_array_equal(gmin[valid], omin[valid])
    np.testing.assert_array_equal(gmax[valid], omax[valid])
    assert (gmin[~valid] == 7.0).all() and (gmax[~valid] == 7.0).all()   # untouched


def test_build_summaries_block_range():
    B, H, N = 2, 2, 40
    d = _dims(B, 4, H, N, 8, 2, 2)
    kv = random_kv(B, H, N, _gen(2)).to(DEV)
    ctx = torch.tensor([N * 16, N * 16], dtype=torch.int32, device=DEV)
    kmin = torch.zeros((B, H, N, 128), dtype=torch.bfloat16, device=DEV)
    kmax = kmin.clone()
    lsk.build_summaries(d, kv, ctx, kmin, kmax, first_block=10, n_blocks=5)
    torch.cuda.synchronize()
    omin, omax = O.block_summaries(kv_split(kv.cpu())[0], ctx.cpu().numpy())
    np.testing.assert_array_equal(f64(kmin)[:, :, 10:15], omin[:, :, 10:15])
    assert (f64(kmin)[:, :, :10] == 0).all() and (f64(kmax)[:, :, 15:] == 0).all()


def test_append_matches_rebuild_and_updates_copies():
    B, H, N, K = 3, 2, 6, 4
    d = _dims(B, 4, H, N, K, 2, 2)
    kv = random_kv(B, H, N, _gen(3))
    host = kv.pin_memory()
    ctx0 = torch.tensor([31, 32, 47], dtype=torch.int32)     # t = 15, 0 (new block), 15
    kmin = torch.zeros((B, H, N, 128), dtype=torch.bfloat16, device=DEV)
    kmax = kmin.clone()
    lsk.build_summaries(d, host, ctx0.to(DEV), kmin, kmax)
    st = torch.full((B, H, K), -1, dtype=torch.int32)
    st[0, 0, 2] = 1          # block of position 31 resident for (0, 0)
    st[2, 1, 0] = 2          # block of position 47 resident for (2, 1)
    st[1, 0, 3] = 2          # block of position 32 resident for (1, 0)
    pool = torch.zeros((B, H, K, 2, 16, 128), dtype=torch.bfloat16)
    for (b, h, s) in [(0, 0, 2), (2, 1, 0), (1, 0, 3)]:
        pool[b, h, s] = kv[b, h, st[b, h, s]]
    pool_d = pool.to(DEV)
    g = _gen(4)
    k_new = (torch.randn(B, H, 128, generator=g) * 3).to(torch.bfloat16)
    v_new = torch.randn(B, H, 128, generator=g).to(torch.bfloat16)
    ctx_out = torch.zeros(B, dtype=torch.int32, device=DEV)
    lsk.append_kv(d, k_new.to(DEV), v_new.to(DEV), ctx0.to(DEV), ctx_out, host, kmin, kmax,
                  st.to(DEV), pool_d)
    torch.cuda.synchronize()
    assert ctx_out.cpu().tolist() == (ctx0 + 1).tolist()
    grown = kv.clone()
    for b in range(B):
        n, t = divmod(int(ctx0[b]), 16)
        grown[b, :, n, 0, t] = k_new[b]
        grown[b, :, n, 1, t] = v_new[b]
    assert torch.equal(host, grown)                            # host KV written through the mapping
    omin, omax = O.block_summaries(kv_split(grown)[0], (ctx0 + 1).numpy())
    valid = ~np.isnan(omin)
    np.testing.assert_array_equal(f64(kmin)[valid], omin[valid])
    np.testing.assert_array_equal(f64(kmax)[valid], omax[valid])
    pool_h = pool_d.cpu()
    for (b, h, s) in [(0, 0, 2), (2, 1, 0), (1, 0, 3)]:
        assert torch.equal(pool_h[b, h, s], grown[b, h, st[b, h, s]])
    assert torch.equal(pool_h[0, 1], pool[0, 1])               # non-resident heads untouched


# ----------------------------------------------------------------- scores
@pytest.mark.parametrize("Hq,Hkv,Qn,N", [(8, 2, 5, 300), (32, 8, 5, 130), (64, 8, 8, 200),
                                         (8, 8, 1, 129), (12, 4, 3, 257), (16, 2, 4, 64)])
def test_lookahead_scores(Hq, Hkv, Qn, N):
    B = 2
    d = _dims(B, Hq, Hkv, N, min(32, N), Qn, 4)
    g = _gen(10 + Hq + Qn)
    kv = random_kv(B, Hkv, N, g)
    q = (torch.randn(B, Qn, Hq, 128, generator=g) * 1.5).to(torch.bfloat16)
    ctx = torch.tensor([N * 16 - 3, (N // 2) * 16 + 1], dtype=torch.int32)
    kmin = torch.zeros((B, Hkv, N, 128), dtype=torch.bfloat16, device=DEV)
    kmax = kmin.clone()
    lsk.build_summaries(d, kv.to(DEV), ctx.to(DEV), kmin, kmax)
    scores = torch.full((B, Hkv, N), 12345.0, device=DEV)
    lsk.lookahead_scores(d, q.to(DEV), kmin, kmax, ctx.to(DEV), scores)
    torch.cuda.synchronize()
    ref = O.lookahead_scores(f64(q), f64(kmin), f64(kmax), ctx.numpy(), 16)
    got = scores.cpu().numpy()
    nv = O.n_valid_blocks(ctx.numpy(), 16)
    for b in range(B):
        r, gg = ref[:, :, :nv[b]][b], got[:, :, :nv[b]][b]
        # every term max(q*kmin, q*kmax) is >= 0 when kmin <= 0 <= kmax, so the sums
        # do not cancel and the fp32 accumulation error stays relative: the bare
        # 1e-5 tie window is the bound, with no absolute slack
        np.testing.assert_allclose(gg, r, rtol=SCORE_REL, atol=0)
        assert (got[b, :, nv[b]:] == 12345.0).all()


# ----------------------------------------------------------------- select
@pytest.mark.parametrize("N,K,nv_blocks", [(300, 32, 300), (300, 32, 20), (2048, 128, 2048),
                                           (8192, 256, 8000), (64, 64, 64), (1000, 1000, 999),
                                           (301, 32, 297), (4097, 128, 4097)])
def test_select_topk_bit_exact(N, K, nv_blocks):
    B, H = 2, 3
    d = _dims(B, 6, H, N, K, 2, 1)
    g = _gen(N + K)
    s = torch.randint(-50, 50, (B, H, N), generator=g).float() * 0.25     # many exact ties
    s[0, 0, ::3] = 0.0
    s[0, 0, 1::3] = -0.0
    s[1] = torch.randn(H, N, generator=g)
    ctx = torch.tensor([nv_blocks * 16, nv_blocks * 16 - 15], dtype=torch.int32)
    sel = torch.empty((B, H, K), dtype=torch.int32, device=DEV)
    sel_s = torch.empty((B, H, K), device=DEV)
    lsk.select_topk(d, s.to(DEV), ctx.to(DEV), sel, sel_s)
    torch.cuda.synchronize()
    ref, ref_s = O.select_topk(s.numpy(), ctx.numpy(), K, 16)
    np.testing.assert_array_equal(np_i32(sel), ref)
    np.testing.assert_array_equal(sel_s.cpu().numpy(), ref_s)


def test_score_select_matches_oracle_up_to_ties():
    w = W.WORKLOADS["tiny"]
    d = lsk.dims_for(w)
    kv = W.make_host_kv(w)
    ctx = W.initial_ctx_len(w)
    q = W.QueryStream(w).next()
    kmin = torch.zeros((w.batch, w.n_kv_heads, w.max_blocks, 128), dtype=torch.bfloat16, device=DEV)
    kmax = kmin.clone()
    lsk.build_summaries(d, kv.pin_memory(), ctx.to(DEV), kmin, kmax)
    ws = torch.zeros(lsk.workspace_bytes(d), dtype=torch.uint8, device=DEV)
    sel = torch.empty((w.batch, w.n_kv_heads, w.budget_blocks), dtype=torch.int32, device=DEV)
    lsk.score_select(d, q.to(DEV), kmin, kmax, ctx.to(DEV), sel, None, ws)
    torch.cuda.synchronize()
    keys, _ = kv_split(kv)
    omin, omax = O.block_summaries(keys, ctx.numpy())
    sc = O.lookahead_scores(f64(q), omin, omax, ctx.numpy(), 16)
    ref, _ = O.select_topk(sc, ctx.numpy(), w.budget_blocks, 16)
    assert_selection_matches(np_i32(sel), ref, sc, ctx.numpy(), w.budget_blocks)
    planted = W.planted_positions(w, 0)[0].numpy()
    got = np_i32(sel)
    for h in range(w.n_kv_heads):
        assert set(planted[0, h].tolist()) <= set(got[0, h].tolist())


# ------------------------------------------------------------------- plan
def test_plan_hand_worked_golden():
    from tests.test_oracle import _read_plan_golden
    st = torch.full((1, 1, 3), -1, dtype=torch.int32, device=DEV)
    lu = torch.full((1, 1, 3), -1, dtype=torch.int32, device=DEV)
    for (step,), (cap,), sel, st_after, lu_after, f_slot, f_block in _read_plan_golden():
        d = _dims(1, 1, 1, 6, 3, 1, cap)
        c = max(cap, 1)
        fs = torch.full((1, 1, c), -7, dtype=torch.int32, device=DEV)
        fb = fs.clone()
        nf = torch.full((1, 1), -7, dtype=torch.int32, device=DEV)
        lsk.plan_fetch(d, torch.tensor([[sel]], dtype=torch.int32, device=DEV), st, lu, step, fs, fb, nf)
        torch.cuda.synchronize()
        assert st.cpu()[0, 0].tolist() == st_after and lu.cpu()[0, 0].tolist() == lu_after, step
        n = int(nf.item())
        assert fs.cpu()[0, 0, :n].tolist() == f_slot and fb.cpu()[0, 0, :n].tolist() == f_block


@pytest.mark.parametrize("K,C,N", [(8, 3, 40), (128, 16, 2048), (256, 32, 8192), (1000, 7, 4000), (33, 0, 99)])
def test_plan_fetch_bit_exact_random(K, C, N):
    B, H = 3, 2
    d = _dims(B, 2, H, N, K, 2, C)
    rng = np.random.default_rng(K + C)
    st = np.full((B, H, K), -1, dtype=np.int32)
    lu = np.full((B, H, K), -1, dtype=np.int32)
    st_d = torch.from_numpy(st).to(DEV)
    lu_d = torch.from_numpy(lu).to(DEV)
    c = max(C, 1)
    fs = torch.empty((B, H, c), dtype=torch.int32, device=DEV)
    fb = torch.empty_like(fs)
    nf = torch.empty((B, H), dtype=torch.int32, device=DEV)
    for step in range(12):
        sel = np.full((B, H, K), -1, dtype=np.int32)
        for b in range(B):
            for h in range(H):
                m = int(rng.integers(1, K + 1))
                # reuse part of the resident set so hits, stale and free slots all occur
                res = [x for x in st[b, h] if x >= 0]
                keep = list(rng.permutation(res)[: m // 2]) if res else []
                rest = [x for x in rng.permutation(N) if x not in set(keep)][: m - len(keep)]
                sel[b, h, :m] = np.array(rng.permutation(keep + rest), dtype=np.int32)
        plan = O.plan_fetch(sel, st, lu, step, C)
        lsk.plan_fetch(d, torch.from_numpy(sel).to(DEV), st_d, lu_d, step, fs, fb, nf)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(np_i32(st_d), plan["slot_table"])
        np.testing.assert_array_equal(np_i32(lu_d), plan["last_used"])
        np.testing.assert_array_equal(np_i32(nf), plan["n_fetch"])
        if C:
            np.testing.assert_array_equal(np_i32(fs), plan["fetch_slot"])
            np.testing.assert_array_equal(np_i32(fb), plan["fetch_block"])
        st, lu = plan["slot_table"], plan["last_used"]


# ------------------------------------------- scores + top-K + plan, fused
@pytest.mark.parametrize("Hq,Hkv,Qn,N,K,C,victims", [(8, 2, 5, 300, 32, 6, "lru"), (32, 8, 5, 1000, 128, 16, "lru"),
                                                     (64, 8, 8, 700, 128, 16, "score"), (12, 4, 3, 257, 64, 64, "score"),
                                                     (8, 8, 1, 129, 16, 0, "lru"), (16, 2, 4, 4096, 1024, 40, "lru")])
def test_score_select_plan_matches_separate_kernels_and_oracle(Hq, Hkv, Qn, N, K, C, victims):
    """The one-launch scores + top-K + plan against the three separate
    kernels (bit for bit: selection, selected scores, slot table, recency,
    fetch lists) and against the oracle (selection under the tie rule, plan
    bit-exact on the GPU's selection), over several steps of a random decode
    state, with the step number given by value and read from device memory
    on alternate steps.  Sequences cover a context that fits the budget, one
    with no context at all, and ragged last tiles."""
    B = 3
    d = _dims(B, Hq, Hkv, N, K, Qn, C)
    g = _gen(500 + N + K)
    kv = random_kv(B, Hkv, N, g)
    ctx = torch.tensor([N * 16 - 7, min(N, K) * 16 - 20, 0], dtype=torch.int32)
    ctx_d = ctx.to(DEV)
    kmin = torch.zeros((B, Hkv, N, 128), dtype=torch.bfloat16, device=DEV)
    kmax = kmin.clone()
    lsk.build_summaries(d, kv.to(DEV), ctx_d, kmin, kmax)
    ws = torch.zeros(lsk.workspace_bytes(d), dtype=torch.uint8, device=DEV)
    ws2 = torch.zeros_like(ws)
    okmin, okmax = f64(kmin), f64(kmax)
    c = max(C, 1)
    # fused (F) and separate (S) states, both starting from the same random residency
    rng = np.random.default_rng(N + K)
    st0 = np.full((B, Hkv, K), -1, dtype=np.int32)
    for b in range(B):
        nvb = int(O.n_valid_blocks(ctx.numpy(), 16)[b])
        for h in range(Hkv):
            ids = rng.permutation(max(nvb, 1))[: rng.integers(0, min(K, nvb) + 1)] if nvb else []
            st0[b, h, :len(ids)] = ids
            st0[b, h] = rng.permutation(st0[b, h])
    lu0 = np.where(st0 >= 0, rng.integers(-1, 5, size=st0.shape), -1).astype(np.int32)
    F = {k: torch.from_numpy(v.copy()).to(DEV) for k, v in (("st", st0), ("lu", lu0))}
    S = {k: torch.from_numpy(v.copy()).to(DEV) for k, v in (("st", st0), ("lu", lu0))}
    for X in (F, S):
        X.update(sel=torch.empty((B, Hkv, K), dtype=torch.int32, device=DEV),
                 sel_score=torch.empty((B, Hkv, K), device=DEV),
                 fs=torch.full((B, Hkv, c), -9, dtype=torch.int32, device=DEV),
                 fb=torch.full((B, Hkv, c), -9, dtype=torch.int32, device=DEV),
                 nf=torch.full((B, Hkv), -9, dtype=torch.int32, device=DEV),
                 scores=torch.zeros((B, Hkv, N), device=DEV))
    step_dev = torch.zeros(4, dtype=torch.int32, device=DEV)
    st, lu = st0, lu0
    for step in range(5, 10):
        q = (torch.randn(B, Qn, Hq, 128, generator=g) * 1.3).to(torch.bfloat16)
        qd = q.to(DEV)
        scored = victims == "score"
        step_dev.fill_(step)
        lsk.score_select_plan(d, qd, kmin, kmax, ctx_d, F["sel"], F["sel_score"], F["scores"] if scored else None,
                              F["st"], F["lu"], -1 if step % 2 else step, step_dev if step % 2 else None, F["fs"],
                              F["fb"], F["nf"], ws)
        if scored:
            lsk.lookahead_scores(d, qd, kmin, kmax, ctx_d, S["scores"])
            lsk.select_topk(d, S["scores"], ctx_d, S["sel"], S["sel_score"])
            lsk.plan_fetch_scored(d, S["sel"], S["scores"], S["st"], S["lu"], step, S["fs"], S["fb"], S["nf"])
        else:
            lsk.score_select(d, qd, kmin, kmax, ctx_d, S["sel"], S["sel_score"], ws2)
            lsk.plan_fetch(d, S["sel"], S["st"], S["lu"], step, S["fs"], S["fb"], S["nf"])
        torch.cuda.synchronize()
        nf_np = np_i32(F["nf"])
        for key in ("sel", "sel_score", "st", "lu", "nf"):
            assert torch.equal(F[key], S[key]), f"{key} differs from the separate kernels at step {step}"
        if C:
            for b in range(B):
                for h in range(Hkv):
                    n = nf_np[b, h]
                    assert torch.equal(F["fs"][b, h, :C], S["fs"][b, h, :C]) and n <= C
                    assert torch.equal(F["fb"][b, h, :C], S["fb"][b, h, :C])
        sc = O.lookahead_scores(f64(q), okmin, okmax, ctx.numpy(), 16)
        ref_sel, _ = O.select_topk(sc, ctx.numpy(), K, 16)
        sel = np_i32(F["sel"])
        assert_selection_matches(sel, ref_sel, sc, ctx.numpy(), K)
        assert (sel[2] == -1).all()                                         # no context: nothing selected
        plan = O.plan_fetch(sel, st, lu, step, C, scores=F["scores"].cpu().numpy() if scored else None)
        np.testing.assert_array_equal(np_i32(F["st"]), plan["slot_table"])
        np.testing.assert_array_equal(np_i32(F["lu"]), plan["last_used"])
        np.testing.assert_array_equal(nf_np, plan["n_fetch"])
        if C:
            np.testing.assert_array_equal(np_i32(F["fs"])[..., :C], plan["fetch_slot"])
            np.testing.assert_array_equal(np_i32(F["fb"])[..., :C], plan["fetch_block"])
        st, lu = plan["slot_table"], plan["last_used"]


@pytest.mark.parametrize("B,Hq,Hkv,Qn,N,K,C,victims", [
    (12, 32, 8, 5, 600, 128, 16, "lru"),      # 96 units: whole units, keys handed over in shared memory
    (10, 64, 8, 8, 300, 64, 8, "score"),      # 80 units, whole, score-ordered victims
    (3, 16, 2, 2, 8192, 128, 8, "lru"),       # 6 units of 8192 blocks: many chunks a unit, 64 keys a thread
    (3, 8, 2, 2, 9000, 64, 8, "lru"),         # more keys than the registers hold: shared-memory selection
])
def test_score_select_plan_modes(B, Hq, Hkv, Qn, N, K, C, victims):
    """The fused launch in each of its ways of reaching the selection (whole
    units handed over in shared memory, split units read back from L2 into
    registers, and the shared-memory fallback past 64 keys a thread) against
    the separate kernels bit for bit and against the oracle.  Summaries are
    drawn directly (no KV), with a context that fills every block, one inside
    the budget, one empty, and random lengths for the rest."""
    d = _dims(B, Hq, Hkv, N, K, Qn, C)
    g = _gen(900 + N + K + B)
    kmin_h = (torch.randn(B, Hkv, N, 128, generator=g) - 0.5).to(torch.bfloat16)
    kmax_h = (kmin_h.float() + torch.rand(B, Hkv, N, 128, generator=g) * 2).to(torch.bfloat16)
    lens = [N * 16 - 7, min(N, K) * 16 - 20, 0] + [int(x) for x in torch.randint(1, N * 16, (B - 3,), generator=g)]
    ctx = torch.tensor(lens[:B], dtype=torch.int32)
    ctx_d = ctx.to(DEV)
    kmin, kmax = kmin_h.to(DEV), kmax_h.to(DEV)
    ws = torch.zeros(lsk.workspace_bytes(d), dtype=torch.uint8, device=DEV)
    ws2 = torch.zeros_like(ws)
    okmin, okmax = f64(kmin_h), f64(kmax_h)
    rng = np.random.default_rng(N + K + B)
    st0 = np.full((B, Hkv, K), -1, dtype=np.int32)
    nv = O.n_valid_blocks(ctx.numpy(), 16)
    for b in range(B):
        for h in range(Hkv):
            if nv[b]:
                ids = rng.permutation(int(nv[b]))[: rng.integers(0, min(K, int(nv[b])) + 1)]
                st0[b, h, :len(ids)] = ids
                st0[b, h] = rng.permutation(st0[b, h])
    lu0 = np.where(st0 >= 0, rng.integers(-1, 5, size=st0.shape), -1).astype(np.int32)
    F = {k: torch.from_numpy(v.copy()).to(DEV) for k, v in (("st", st0), ("lu", lu0))}
    S = {k: torch.from_numpy(v.copy()).to(DEV) for k, v in (("st", st0), ("lu", lu0))}
    for X in (F, S):
        X.update(sel=torch.empty((B, Hkv, K), dtype=torch.int32, device=DEV),
                 sel_score=torch.empty((B, Hkv, K), device=DEV),
                 fs=torch.full((B, Hkv, max(C, 1)), -9, dtype=torch.int32, device=DEV),
                 fb=torch.full((B, Hkv, max(C, 1)), -9, dtype=torch.int32, device=DEV),
                 nf=torch.full((B, Hkv), -9, dtype=torch.int32, device=DEV),
                 scores=torch.zeros((B, Hkv, N), device=DEV))
    scored = victims == "score"
    st, lu = st0, lu0
    for step in range(5, 8):
        q = (torch.randn(B, Qn, Hq, 128, generator=g) * 1.3).to(torch.bfloat16)
        qd = q.to(DEV)
        lsk.score_select_plan(d, qd, kmin, kmax, ctx_d, F["sel"], F["sel_score"], F["scores"] if scored else None,
                              F["st"], F["lu"], step, None, F["fs"], F["fb"], F["nf"], ws)
        if scored:
            lsk.lookahead_scores(d, qd, kmin, kmax, ctx_d, S["scores"])
            lsk.select_topk(d, S["scores"], ctx_d, S["sel"], S["sel_score"])
            lsk.plan_fetch_scored(d, S["sel"], S["scores"], S["st"], S["lu"], step, S["fs"], S["fb"], S["nf"])
        else:
            lsk.score_select(d, qd, kmin, kmax, ctx_d, S["sel"], S["sel_score"], ws2)
            lsk.plan_fetch(d, S["sel"], S["st"], S["lu"], step, S["fs"], S["fb"], S["nf"])
        torch.cuda.synchronize()
        assert lsk.read_device_error(clear=True) == 0
        for key in ("sel", "sel_score", "st", "lu", "nf"):
            assert torch.equal(F[key], S[key]), f"{key} differs from the separate kernels at step {step}"
        for b in range(B):
            for h in range(Hkv):
                n = int(np_i32(F["nf"])[b, h])
                assert n <= C
                assert torch.equal(F["fs"][b, h, :n], S["fs"][b, h, :n])
                assert torch.equal(F["fb"][b, h, :n], S["fb"][b, h, :n])
        sc = O.lookahead_scores(f64(q), okmin, okmax, ctx.numpy(), 16)
        ref_sel, _ = O.select_topk(sc, ctx.numpy(), K, 16)
        sel = np_i32(F["sel"])
        assert_selection_matches(sel, ref_sel, sc, ctx.numpy(), K)
        assert (sel[2] == -1).all()
        plan = O.plan_fetch(sel, st, lu, step, C, scores=F["scores"].cpu().numpy() if scored else None)
        np.testing.assert_array_equal(np_i32(F["st"]), plan["slot_table"])
        np.testing.assert_array_equal(np_i32(F["lu"]), plan["last_used"])
        np.testing.assert_array_equal(np_i32(F["nf"]), plan["n_fetch"])
        st, lu = plan["slot_table"], plan["last_used"]


# --------------------------------------------------------------- prefetch
def test_prefetch_bytes_exact():
    B, H, N, K, C = 2, 3, 50, 16, 6
    d = _dims(B, 3, H, N, K, 1, C)
    kv = random_kv(B, H, N, _gen(5)).pin_memory()
    rng = np.random.default_rng(5)
    fs = np.full((B, H, C), -1, dtype=np.int32)
    fb = np.full((B, H, C), -1, dtype=np.int32)
    nf = rng.integers(0, C + 1, size=(B, H)).astype(np.int32)
    for b in range(B):
        for h in range(H):
            n = nf[b, h]
            fs[b, h, :n] = rng.permutation(K)[:n]
            fb[b, h, :n] = rng.permutation(N)[:n]
    pool = torch.randint(-30000, 30000, (B, H, K, 2, 16, 128), dtype=torch.int16).view(torch.bfloat16)
    pool_d = pool.to(DEV)
    lsk.prefetch(d, kv, torch.from_numpy(fs).to(DEV), torch.from_numpy(fb).to(DEV),
                 torch.from_numpy(nf).to(DEV), pool_d)
    torch.cuda.synchronize()
    ref = O.prefetch(W.bf16_bits(kv), W.bf16_bits(pool), fs, fb, nf)
    np.testing.assert_array_equal(W.bf16_bits(pool_d), ref)


def test_prefetch_rejects_device_memory_as_host_kv():
    d = _dims(1, 1, 1, 16, 4, 1, 2)
    t = torch.zeros(16 * 4096, dtype=torch.bfloat16, device=DEV)
    i = torch.zeros(4, dtype=torch.int32, device=DEV)
    with pytest.raises(lsk.OasisError) as e:
        lsk.prefetch(d, t, i, i, i, t)
    assert e.value.code == lsk.ENOTMAPPED


# -------------------------------------------------------------- attention
@pytest.mark.parametrize("Hq,Hkv,Qn,K", [(8, 2, 5, 32), (32, 8, 5, 128), (64, 8, 8, 128), (4, 4, 1, 20),
                                         (16, 2, 2, 40), (24, 4, 6, 56), (40, 8, 7, 16), (8, 1, 8, 200)])
def test_sparse_attention(Hq, Hkv, Qn, K):
    B, N = 2, 3 * K + 5
    d = _dims(B, Hq, Hkv, N, K, Qn, 4)
    g = _gen(100 + Hq * Qn + K)
    kv = random_kv(B, Hkv, N, g)
    q = torch.randn(B, Qn, Hq, 128, generator=g).to(torch.bfloat16)
    ctx = torch.tensor([N * 16 - 9, K * 16], dtype=torch.int32)
    rng = np.random.default_rng(K)
    st = np.full((B, Hkv, K), -1, dtype=np.int32)
    for b in range(B):
        nvb = int(O.n_valid_blocks(ctx.numpy(), 16)[b])
        for h in range(Hkv):
            occ = rng.random(K) < 0.8
            blocks = rng.permutation(N)[:K]          # includes blocks beyond the context
            st[b, h] = np.where(occ, blocks, -1)
            st[b, h][st[b, h] == nvb - 1] = -1
            st[b, h, 0] = nvb - 1                    # the partial last block
    if Hkv > 1:
        st[1, 1] = -1                                # a head with nothing resident
    pool = torch.zeros((B, Hkv, K, 2, 16, 128), dtype=torch.bfloat16)
    for b in range(B):
        for h in range(Hkv):
            for s in range(K):
                if st[b, h, s] >= 0:
                    pool[b, h, s] = kv[b, h, st[b, h, s]]
    scale = 1 / math.sqrt(128)
    out = torch.empty((B, Qn, Hq, 128), device=DEV)
    lse = torch.empty((B, Qn, Hq), device=DEV)
    ws = torch.zeros(lsk.workspace_bytes(d), dtype=torch.uint8, device=DEV)
    pool_clean = pool
    pk, pv = kv_split(pool_clean)
    for _ in range(2):                                # second call reuses the zeroed counters
        lsk.sparse_attn(d, q.to(DEV), pool_clean.to(DEV), torch.from_numpy(st).to(DEV), ctx.to(DEV),
                        scale, out, lse, ws)
        torch.cuda.synchronize()
        o_ref, lse_ref = O.sparse_attention(f64(q), pk, pv, st, ctx.numpy(), scale)
        assert_attention_close(out, lse, o_ref, lse_ref)


@pytest.mark.parametrize("B,Hq,Hkv,Qn,K", [(40, 32, 4, 8, 16),     # 64 rows, 160 whole units
                                           (35, 16, 2, 8, 128),    # 64 rows, 70 units of 2 chunks
                                           (40, 16, 4, 5, 16)])    # 20 rows, 160 whole units
def test_sparse_attention_more_chunks_than_ctas(B, Hq, Hkv, Qn, K):
    """More chunks than the launch has CTAs (at most one per SM, less the
    gather's 16), so CTAs take further chunks from the counter: a chunk's
    query rows land in the buffer the CTA's previous chunk read (the only one
    with 64 rows) once that chunk's S^T products are done, and split units
    are merged by whichever of their chunks finishes last."""
    N = K + 7
    d = _dims(B, Hq, Hkv, N, K, Qn, 4)
    g = _gen(900 + B + K)
    kv = random_kv(B, Hkv, N, g)
    q = torch.randn(B, Qn, Hq, 128, generator=g).to(torch.bfloat16)
    rng = np.random.default_rng(B * K)
    ctx = torch.from_numpy(rng.integers(K * 16 - 40, N * 16 + 1, size=B).astype(np.int32))
    nvb = O.n_valid_blocks(ctx.numpy(), 16)
    st = np.full((B, Hkv, K), -1, dtype=np.int32)
    for b in range(B):
        for h in range(Hkv):
            blocks = rng.permutation(N)[:K]          # includes blocks beyond the context
            st[b, h] = np.where(rng.random(K) < 0.85, blocks, -1)
            st[b, h][st[b, h] == nvb[b] - 1] = -1
            st[b, h, rng.integers(K)] = nvb[b] - 1   # the partial last block
    st[B - 1, Hkv - 1] = -1                          # a head with nothing resident
    idx = torch.from_numpy(np.maximum(st, 0)).long()
    pool = kv[torch.arange(B)[:, None, None], torch.arange(Hkv)[None, :, None], idx]
    pool[torch.from_numpy(st < 0)] = 0
    scale = 1 / math.sqrt(128)
    out = torch.empty((B, Qn, Hq, 128), device=DEV)
    lse = torch.empty((B, Qn, Hq), device=DEV)
    ws = torch.zeros(lsk.workspace_bytes(d), dtype=torch.uint8, device=DEV)
    pk, pv = kv_split(pool)
    o_ref, lse_ref = O.sparse_attention(f64(q), pk, pv, st, ctx.numpy(), scale)
    for _ in range(2):                                # second call reuses the zeroed counters
        out.fill_(float("nan"))
        lsk.sparse_attn(d, q.to(DEV), pool.to(DEV), torch.from_numpy(st).to(DEV), ctx.to(DEV),
                        scale, out, lse, ws)
        torch.cuda.synchronize()
        assert_attention_close(out, lse, o_ref, lse_ref)


def test_sparse_attention_masks_garbage_beyond_context():
    """Values of tokens beyond ctx_len (NaN here) never reach the output."""
    B, Hq, Hkv, K, N = 1, 4, 1, 8, 20
    d = _dims(B, Hq, Hkv, N, K, 2, 2)
    g = _gen(7)
    kv = random_kv(B, Hkv, N, g)
    q = torch.randn(B, 2, Hq, 128, generator=g).to(torch.bfloat16)
    ctx = torch.tensor([5 * 16 + 3], dtype=torch.int32)
    st = np.array([[[5, 0, 1, -1, 2, 3, -1, 9]]], dtype=np.int32)
    pool = torch.zeros((B, Hkv, K, 2, 16, 128), dtype=torch.bfloat16)
    for s in range(K):
        if st[0, 0, s] >= 0:
            pool[0, 0, s] = kv[0, 0, st[0, 0, s]]
    clean = pool.clone()
    pool[0, 0, 0, :, 3:] = float("nan")             # block 5 holds 3 valid tokens (80..82)
    pool[0, 0, 7] = float("nan")                    # block 9 is beyond the context
    out = torch.empty((B, 2, Hq, 128), device=DEV)
    lse = torch.empty((B, 2, Hq), device=DEV)
    ws = torch.zeros(lsk.workspace_bytes(d), dtype=torch.uint8, device=DEV)
    lsk.sparse_attn(d, q.to(DEV), pool.to(DEV), torch.from_numpy(st).to(DEV), ctx.to(DEV), 0.1, out, lse, ws)
    torch.cuda.synchronize()
    pk, pv = kv_split(clean)
    o_ref, lse_ref = O.sparse_attention(f64(q), pk, pv, st, ctx.numpy(), 0.1)
    assert_attention_close(out, lse, o_ref, lse_ref)


def test_sparse_attention_full_budget_is_dense():
    """Budget covering the context: sparse attention equals dense attention."""
    B, Hq, Hkv, N = 2, 16, 4, 24
    K = N
    d = _dims(B, Hq, Hkv, N, K, 3, 4)
    g = _gen(8)
    kv = random_kv(B, Hkv, N, g)
    q = torch.randn(B, 3, Hq, 128, generator=g).to(torch.bfloat16)
    ctx = torch.tensor([N * 16, N * 16 - 20], dtype=torch.int32)
    st = np.stack([np.stack([np.random.default_rng(b * 7 + h).permutation(N) for h in range(Hkv)])
                   for b in range(B)]).astype(np.int32)
    pool = torch.stack([torch.stack([kv[b, h, torch.from_numpy(st[b, h]).long()] for h in range(Hkv)])
                        for b in range(B)])
    out = torch.empty((B, 3, Hq, 128), device=DEV)
    lse = torch.empty((B, 3, Hq), device=DEV)
    ws = torch.zeros(lsk.workspace_bytes(d), dtype=torch.uint8, device=DEV)
    lsk.sparse_attn(d, q.to(DEV), pool.to(DEV), torch.from_numpy(st).to(DEV), ctx.to(DEV), 0.0883883, out,
                    lse, ws)
    torch.cuda.synchronize()
    keys, vals = kv_split(kv)
    o_ref, lse_ref = O.dense_attention(f64(q), keys, vals, ctx.numpy(), 0.0883883)
    assert_attention_close(out, lse, o_ref, lse_ref)


# ------------------------------------------------------------ error word
def test_duplicate_resident_block_sets_error_word_without_fault():
    """A slot table that holds one block in two slots is an invalid state: the
    planner (standalone and inside the fused launch) flags it in the device
    error word and finishes; the other unit's plan is unaffected."""
    B, H, N, K, C = 1, 2, 64, 8, 3
    d = _dims(B, 4, H, N, K, 1, C)
    assert lsk.read_device_error(clear=True) == 0
    st0 = torch.tensor([[[5, 9, 5, -1, 12, -1, 7, -1], [1, 2, 3, -1, -1, -1, -1, -1]]], dtype=torch.int32)
    sel = torch.tensor([[[5, 40, 41, 9, -1, -1, -1, -1], [1, 2, 50, 51, 52, -1, -1, -1]]], dtype=torch.int32, device=DEV)
    st, lu = st0.to(DEV), torch.zeros_like(st0).to(DEV)
    fs = torch.empty((B, H, C), dtype=torch.int32, device=DEV)
    fb = torch.empty_like(fs)
    nf = torch.empty((B, H), dtype=torch.int32, device=DEV)
    lsk.plan_fetch(d, sel, st, lu, 1, fs, fb, nf)
    assert lsk.read_device_error(clear=True) & lsk.DEVERR_DUPLICATE
    # the valid unit: misses 50, 51, 52 into its free slots 3, 4, 5 in slot order
    ref = O.plan_fetch(np_i32(sel)[:, 1:], st0.numpy()[:, 1:], np.zeros((1, 1, K), np.int32), 1, C)
    np.testing.assert_array_equal(np_i32(st)[:, 1:], ref["slot_table"])
    np.testing.assert_array_equal(np_i32(nf)[:, 1:], ref["n_fetch"])
    # the fused launch on the same state
    g = _gen(77)
    q = torch.randn((B, 1, 4, 128), generator=g).to(torch.bfloat16).to(DEV)
    kmin = (torch.randn((B, H, N, 128), generator=g) - 1).to(torch.bfloat16).to(DEV)
    kmax = (kmin.float() + 2).to(torch.bfloat16)
    ctx = torch.tensor([N * 16], dtype=torch.int32, device=DEV)
    ws = torch.zeros(lsk.workspace_bytes(d), dtype=torch.uint8, device=DEV)
    st2, lu2 = st0.to(DEV), torch.zeros_like(st0).to(DEV)
    sel2 = torch.empty_like(sel)
    lsk.score_select_plan(d, q, kmin, kmax, ctx, sel2, None, None, st2, lu2, 1, None, fs, fb, nf, ws)
    assert lsk.read_device_error(clear=True) & lsk.DEVERR_DUPLICATE


def test_out_of_range_ids_set_error_word_without_fault():
    B, H, N, K = 1, 1, 10, 4
    d = _dims(B, 2, H, N, K, 1, 2)
    assert lsk.read_device_error(clear=True) == 0
    st = torch.tensor([[[3, 99, -5, 1]]], dtype=torch.int32, device=DEV)
    lu = torch.zeros_like(st)
    sel = torch.tensor([[[2, 1, 500, -1]]], dtype=torch.int32, device=DEV)
    fs = torch.empty((1, 1, 2), dtype=torch.int32, device=DEV)
    fb = torch.empty_like(fs)
    nf = torch.empty((1, 1), dtype=torch.int32, device=DEV)
    lsk.plan_fetch(d, sel, st, lu, 1, fs, fb, nf)
    assert lsk.read_device_error(clear=True) & lsk.DEVERR_ID_RANGE
    q = torch.zeros((1, 1, 2, 128), dtype=torch.bfloat16, device=DEV)
    pool = torch.zeros((1, 1, K, 2, 16, 128), dtype=torch.bfloat16, device=DEV)
    bad = torch.tensor([[[3, 99, 1, 2]]], dtype=torch.int32, device=DEV)
    ws = torch.zeros(lsk.workspace_bytes(d), dtype=torch.uint8, device=DEV)
    out = torch.empty((1, 1, 2, 128), device=DEV)
    lse = torch.empty((1, 1, 2), device=DEV)
    lsk.sparse_attn(d, q, pool, bad, torch.tensor([160], dtype=torch.int32, device=DEV), 0.1, out, lse, ws)
    assert lsk.read_device_error(clear=True) & lsk.DEVERR_ID_RANGE
    assert torch.isfinite(out).all()
