"""Shared helpers of the GPU parity tests: tensor <-> oracle conversions,
random decode states, and the comparison rules (bit-exact for ids and bytes,
the 1e-5 relative tie window for selections, abs 2e-3 / rel 1e-2 for the
attention output)."""

import numpy as np
import torch

import oracle as O
from lookahead_sparse_kv_b200 import workloads as W

ATOL, RTOL = 2e-3, 1e-2          # attention output / lse
TIE_REL = 1e-5                   # selection boundary tie window (relative to the K-th score)
SCORE_REL = 1e-5                 # tensor-core fp32 accumulation vs fp64-then-fp32


def f64(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> exact float64 numpy."""
    return O.bf16_bits_to_f64(W.bf16_bits(t))


def np_i32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.int32)


def kv_split(host_kv: torch.Tensor):
    """[B,H,N,2,P,D] bf16 -> (keys, values) float64 [B,H,N,P,D]."""
    a = f64(host_kv)
    return a[:, :, :, 0], a[:, :, :, 1]


def random_kv(B, H, N, gen, scale_channels=True, device="cpu"):
    kv = torch.randn(B, H, N, 2, 16, 128, generator=gen, device=device)
    if scale_channels:
        kv[..., :4] *= 8.0
    return kv.to(torch.bfloat16)


def assert_selection_matches(sel_gpu, sel_or, scores_or, ctx, K, P=16, tie=TIE_REL):
    """Selections agree up to the stated tie rule: a block may differ only if
    its oracle score is within `tie` relative of the oracle's K-th score."""
    B, H, _ = sel_or.shape
    nv = O.n_valid_blocks(ctx, P)
    for b in range(B):
        for h in range(H):
            g = [int(x) for x in sel_gpu[b, h] if x >= 0]
            o = [int(x) for x in sel_or[b, h] if x >= 0]
            assert len(g) == len(o) == min(K, int(nv[b])), (b, h, len(g), len(o))
            assert len(set(g)) == len(g)
            if g == o:
                continue
            kth = float(scores_or[b, h, o[-1]])
            win = tie * max(abs(kth), 1e-30)
            for blk in set(g) ^ set(o):
                assert abs(float(scores_or[b, h, blk]) - kth) <= win, (b, h, blk)
            # rank order may differ only between near-equal scores
            s = [float(scores_or[b, h, x]) for x in g]
            for i in range(len(s) - 1):
                assert s[i] >= s[i + 1] - tie * max(abs(s[i]), 1e-30), (b, h, i)


def assert_attention_close(o_gpu, lse_gpu, o_or, lse_or, atol=ATOL, rtol=RTOL):
    o_gpu = o_gpu.detach().cpu().double().numpy()
    lse_gpu = lse_gpu.detach().cpu().double().numpy()
    np.testing.assert_allclose(o_gpu, o_or, atol=atol, rtol=rtol)
    fin = np.isfinite(lse_or)
    assert (np.isfinite(lse_gpu) == fin).all()
    np.testing.assert_allclose(lse_gpu[fin], lse_or[fin], atol=atol, rtol=rtol)


def sampled_units(w, n, seed=0):
    """n distinct (sequence, KV head) units of workload w for sampled checks:
    the first and the last unit of the batch (the last sequence's last KV
    head, where an off-by-one in a unit index would show), the rest seeded."""
    rng = np.random.default_rng(seed)
    total = w.batch * w.n_kv_heads
    picks = [0, total - 1]
    for u in rng.permutation(total):
        if len(picks) >= min(n, total):
            break
        if int(u) not in picks:
            picks.append(int(u))
    return [divmod(u, w.n_kv_heads) for u in picks]
