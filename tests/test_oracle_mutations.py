"""Each plausible mistake planted in a temporary copy of the oracle must make
at least one oracle pin fail.  Runs the pin suite on the mutated copy in a
subprocess; CPU only."""

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "verification row scored": (
        "rows = list(range(1, Qn)) if Qn > 1 else [0]", "rows = list(range(0, Qn))"),
    "kmin term dropped": (
        "np.maximum(qs[:, None, :] * lo[None], qs[:, None, :] * hi[None])", "qs[:, None, :] * hi[None]"),
    "ties to the higher index": (
        "key=lambda n: (-float(s[n]), n)", "key=lambda n: (-float(s[n]), -n)"),
    "most recently used evicted": (
        "stale.sort(key=lambda slot: (int(lu[b, h, slot]), int(st[b, h, slot])))",
        "stale.sort(key=lambda slot: (-int(lu[b, h, slot]), int(st[b, h, slot])))"),
    "stale slots before free ones": ("victims = free + stale", "victims = stale + free"),
    "lowest-ranked misses fetched": (
        "fetch = missing[:min(C, len(missing))]",
        "fetch = missing[-min(C, len(missing)):] if missing and C else []"),
    "masked tokens summarised": ("valid = min(P, ctx - n * P)\n            tokens", "valid = P\n            tokens"),
    "hits not stamped": ("lu[b, h, resident[blk]] = step", "pass"),
    "softmax scale dropped": ("logits = scale * (qh @ kt.T)  ", "logits = (qh @ kt.T)  "),
    "output rows transposed": (
        "reshape(Qn, G, D)\n            lse[b, :, h * G:(h + 1) * G] = (m + np.log(l)).reshape(Qn, G)\n"
        "    return o, lse\n\n\ndef dense_attention",
        "reshape(G, Qn, D).transpose(1, 0, 2)\n"
        "            lse[b, :, h * G:(h + 1) * G] = (m + np.log(l)).reshape(Qn, G)\n"
        "    return o, lse\n\n\ndef dense_attention"),
    # prediction quality, corrective fetch, victim order, residency loss: their own pin files
    "overlap counts repeated ids": (
        "out[i, h] = len(sa & sb)", "out[i, h] = sum(1 for x in b[i, h] if x >= 0 and int(x) in sa)",
        ["test_oracle_prediction.py"]),
    "exact set scored from the drafts": (
        "select_topk(lookahead_scores(qs, kmin, kmax, ctx_len, P, rows=[0]), ctx_len, K, P)",
        "select_topk(lookahead_scores(qs, kmin, kmax, ctx_len, P), ctx_len, K, P)",
        ["test_oracle_prediction.py"]),
    "corrective fetch capped": (
        "plan = plan_fetch(exact, st, lu, step, K)", "plan = plan_fetch(exact, st, lu, step, fetch_cap)",
        ["test_oracle_prediction.py"]),
    "highest-scored stale block evicted": (
        "stale.sort(key=lambda slot: (float(scores[b, h, st[b, h, slot]]), int(st[b, h, slot])))",
        "stale.sort(key=lambda slot: (-float(scores[b, h, st[b, h, slot]]), int(st[b, h, slot])))",
        ["test_oracle_eviction.py"]),
    "lost slots kept": (
        "st[np.asarray(mask, dtype=bool)] = -1", "st = st", ["test_oracle_eviction.py"]),
    # Quest's bound carries no 1/sqrt(D) and takes the max over the query heads (R1)
    "bound scaled by 1/sqrt(D)": ("bound = term.sum(axis=2)                             # [R, n], fp64",
                                  "bound = term.sum(axis=2) / math.sqrt(D)"),
    "bound summed over query heads": ("out[b, h, n0:n1] = bound.max(axis=0).astype(np.float32)",
                                      "out[b, h, n0:n1] = bound.sum(axis=0).astype(np.float32)"),
    "valid blocks rounded down": ("return (ctx + block_tokens - 1) // block_tokens", "return ctx // block_tokens"),
    "gather slot and block swapped": (
        "out[b, h, int(fetch_slot[b, h, i])] = host_kv[b, h, int(fetch_block[b, h, i])]",
        "out[b, h, int(fetch_block[b, h, i]) % out.shape[2]] = host_kv[b, h, int(fetch_slot[b, h, i])]"),
    "append never reopens a block": ("        if t == 0:\n            kmin[b, :, n, :] = k_new[b]",
                                     "        if False:\n            kmin[b, :, n, :] = k_new[b]"),
    "attention sees one token past the context": ("valid = min(P, ctx - blk * P)", "valid = min(P, ctx + 1 - blk * P)"),
    "one block short of the budget": ("            take = order[:K]\n", "            take = order[:K - 1]\n"),
    "one fetch over the cap": ("fetch = missing[:min(C, len(missing))]", "fetch = missing[:min(C + 1, len(missing))]"),
    # under LRU a just-stamped selected resident never sorts first, so only score-ordered victims show it
    "selected residents not protected": (
        "                     if st[b, h, slot] >= 0 and int(st[b, h, slot]) not in in_sel]",
        "                     if st[b, h, slot] >= 0]",
        ["test_oracle.py", "test_oracle_eviction.py"]),
    # R9: the appended row reaches the resident copy of its block, and the context grows
    "appended row not copied into the resident slot": (
        "                    pool_k[b, h, slot, t] = k_new[b, h]\n", "                    pass\n"),
    "context not grown by an append": ("    return np.asarray(ctx_len, dtype=np.int64) + 1\n",
                                       "    return np.asarray(ctx_len, dtype=np.int64)\n"),
    # Figure 8: attention at step t reads the working set staged at step t-1, not this step's fetch
    "attention over this step's fetch": (
        "        o, lse = sparse_attention(qs, pool_k, pool_v, st, ctx_len, scale)\n"
        "        slot_table_used = st.copy()\n"
        "        if evict_masks is not None:\n"
        "            st = evict_slots(st, evict_masks[t - 1])\n"
        "        sc, sel, sel_score, plan = select_plan_fetch(qs, t)\n",
        "        if evict_masks is not None:\n"
        "            st = evict_slots(st, evict_masks[t - 1])\n"
        "        sc, sel, sel_score, plan = select_plan_fetch(qs, t)\n"
        "        o, lse = sparse_attention(qs, pool_k, pool_v, st, ctx_len, scale)\n"
        "        slot_table_used = st.copy()\n",
        ["test_oracle.py", "test_oracle_prediction.py", "test_oracle_eviction.py"]),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new, *pins = MUTATIONS[name]
    pins = pins[0] if pins else ["test_oracle.py"]
    for sub in ("oracle", "tests", "lookahead_sparse_kv_b200"):
        shutil.copytree(os.path.join(ROOT, sub), tmp_path / sub,
                        ignore=shutil.ignore_patterns("*.so", "__pycache__", "_build"))
    src_path = tmp_path / "oracle" / "oasis_oracle.py"
    src = src_path.read_text()
    assert src.count(old) == 1, f"mutation anchor not found once: {name}"
    src_path.write_text(src.replace(old, new))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider"] +
                       [str(tmp_path / "tests" / f) for f in pins],
                       cwd=tmp_path, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"no pin failed for planted mistake: {name}\n{r.stdout[-2000:]}"
