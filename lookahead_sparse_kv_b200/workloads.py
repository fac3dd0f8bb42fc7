"""Seeded synthetic workloads for the lookahead sparse-KV decode path.

This module only draws random inputs: keys, values and queries shaped like
the OasisKV pages' workloads, plus the workload-level disturbances some
configurations apply (a seeded residency-loss mask, appended token rows).  It
holds none of the method's arithmetic, so both the CUDA path and the CPU
oracle can take their inputs from here without sharing any computation.

Every draw comes from a ``torch.Generator`` seeded from (workload seed,
layer, purpose), on the device the caller names.  CPU and CUDA generators
produce different streams for the same seed; each stream is reproducible on
its own device, and a test always feeds the same bytes to both sides.

Shapes (bf16 unless noted):
  host KV   [B, Hkv, N, 2, P, D]   (K rows then V rows of each 16-token block)
  queries   [B, Qn, Hq, D]         (row 0 verification, rows 1.. drafts)
  ctx_len   [B] int32
"""

from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import torch

HEAD_DIM = 128
BLOCK_TOKENS = 16


@dataclass(frozen=True)
class Workload:
    """One synthetic decode workload (shapes + value distributions)."""

    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    context: int                 # context tokens at the first decode step
    max_blocks: int              # N: block capacity per (sequence, KV head)
    budget_blocks: int           # K: token budget / P
    n_queries: int               # 1 verification + k drafts
    fetch_cap: int               # C: blocks fetched per (sequence, head) per step
    layers: int = 1
    steps: int = 8
    head_dim: int = HEAD_DIM
    block_tokens: int = BLOCK_TOKENS
    outlier_channels: int = 4    # per KV head, scaled in both K and V
    outlier_scale: float = 8.0
    planted_blocks: int = 0      # relevant blocks per (sequence, head) and group
    planted_groups: int = 1      # >1: groups keyed to their own directions
    hop_every: int = 0           # steps between switches of the query direction group
    key_dist: str = "normal"     # "normal" | "student_t3"
    ar_rho: float = 0.0          # AR(1) coefficient of the query drift term (0 = no drift)
    drift_scale: float = 0.3     # size of the AR(1) drift term relative to the mean
    query_mean_scale: float = 1.0
    query_noise: float = 0.5
    planted_key_scale: float = 0.5
    evict_prob: float = 0.0      # per-step probability that a resident slot is lost
    append: bool = False         # one new token per sequence per step
    draft_lead: bool = False     # draft row j follows the query mean j steps ahead (see QueryStream)
    seed: int = 20260807

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_drafts(self) -> int:
        return self.n_queries - 1

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    # sizes -----------------------------------------------------------
    @property
    def block_bytes(self) -> int:
        return 2 * self.block_tokens * self.head_dim * 2

    def host_kv_bytes(self) -> int:
        return self.batch * self.n_kv_heads * self.max_blocks * self.block_bytes

    def pool_bytes(self) -> int:
        return self.batch * self.n_kv_heads * self.budget_blocks * self.block_bytes

    def summary_bytes(self) -> int:
        return 2 * self.batch * self.n_kv_heads * self.max_blocks * self.head_dim * 2


def _blocks(tokens: int) -> int:
    return (tokens + BLOCK_TOKENS - 1) // BLOCK_TOKENS


# The five workloads of the pages' evaluation, as synthetic shapes.
WORKLOADS = {
    # Tiny single-layer case with planted relevant blocks.
    "tiny": Workload("tiny", batch=1, n_q_heads=8, n_kv_heads=2, context=4096,
                     max_blocks=_blocks(4096), budget_blocks=32, n_queries=5,
                     fetch_cap=8, steps=8, planted_blocks=6),
    # Llama-3.1-8B attention layer at 32K, AR(1) query drift.
    "llama8b_32k": Workload("llama8b_32k", batch=16, n_q_heads=32, n_kv_heads=8,
                            context=32768, max_blocks=_blocks(32768), budget_blocks=128,
                            n_queries=5, fetch_cap=16, steps=64, ar_rho=0.9,
                            query_noise=0.05),
    # Qwen3-8B reasoning decode: 36 layers, context grows 1K -> 17K by appends.
    "qwen8b_reasoning": Workload("qwen8b_reasoning", batch=64, n_q_heads=32, n_kv_heads=8,
                                 context=1024, max_blocks=_blocks(17408), budget_blocks=128,
                                 n_queries=5, fetch_cap=8, layers=36, steps=32,
                                 ar_rho=0.9, query_noise=0.05, append=True),
    # Qwen3-32B stack at 32K: 64 layers, 1+7 queries, 10% residency loss per step.
    "qwen32b_32k": Workload("qwen32b_32k", batch=16, n_q_heads=64, n_kv_heads=8,
                            context=32768, max_blocks=_blocks(32768), budget_blocks=128,
                            n_queries=8, fetch_cap=16, layers=64, steps=16,
                            ar_rho=0.9, query_noise=0.05, evict_prob=0.1),
    # The 32K Llama layer with drafts that lead the verification query (the
    # prediction-quality and corrective-fetch measurements).
    "llama8b_32k_lead": Workload("llama8b_32k_lead", batch=16, n_q_heads=32, n_kv_heads=8,
                                 context=32768, max_blocks=_blocks(32768), budget_blocks=128,
                                 n_queries=5, fetch_cap=16, steps=64, ar_rho=0.9,
                                 query_noise=0.05, draft_lead=True),
    # 128K stress: heavy-tailed keys, planted groups hopping every 64 steps.
    "longctx_128k": Workload("longctx_128k", batch=8, n_q_heads=32, n_kv_heads=8,
                             context=131072, max_blocks=_blocks(131072), budget_blocks=128,
                             n_queries=5, fetch_cap=16, steps=256, key_dist="student_t3",
                             planted_blocks=6, planted_groups=4, hop_every=64),
}


def _gen(w: Workload, layer: int, purpose: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(w.seed + 100 * (purpose + 1) + 10007 * layer)
    return g


_P_KV, _P_DIR, _P_QUERY, _P_PLANT, _P_EVICT, _P_APPEND, _P_OUTLIER = range(7)


def outlier_channels(w: Workload, layer: int) -> torch.Tensor:
    """Seeded outlier channel indices, int64 [Hkv, outlier_channels] (CPU)."""
    g = _gen(w, layer, _P_OUTLIER, "cpu")
    return torch.stack([torch.randperm(w.head_dim, generator=g)[: w.outlier_channels]
                        for _ in range(w.n_kv_heads)])


def _channel_scale(w: Workload, layer: int, device) -> torch.Tensor:
    """Per (KV head, channel) multiplier: outlier_scale on outlier channels, else 1."""
    scale = torch.ones(w.n_kv_heads, w.head_dim)
    idx = outlier_channels(w, layer)
    for h in range(w.n_kv_heads):
        scale[h, idx[h]] = w.outlier_scale
    return scale.to(device)


def _draw_keys(w: Workload, shape, g: torch.Generator, device) -> torch.Tensor:
    x = torch.randn(shape, generator=g, device=device)
    if w.key_dist == "student_t3":
        chi2 = torch.randn((3,) + tuple(shape), generator=g, device=device).pow_(2).sum(0)
        x = x / torch.sqrt(chi2 / 3.0)
    return x


def mean_directions(w: Workload, layer: int, device="cpu") -> torch.Tensor:
    """Base query mean directions u, fp32 [groups, B, Hkv, D] ~ N(0, I)."""
    g = _gen(w, layer, _P_DIR, device)
    return torch.randn(max(1, w.planted_groups), w.batch, w.n_kv_heads, w.head_dim,
                       generator=g, device=device) * w.query_mean_scale


def planted_positions(w: Workload, layer: int) -> torch.Tensor:
    """Planted block ids, int64 [groups, B, Hkv, planted_blocks] (CPU); all distinct
    within a (b, h) and inside the first ``context`` tokens."""
    g = _gen(w, layer, _P_PLANT, "cpu")
    nb = _blocks(w.context)
    total = max(1, w.planted_groups) * w.planted_blocks
    out = torch.empty(w.batch, w.n_kv_heads, total, dtype=torch.int64)
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            out[b, h] = torch.randperm(nb, generator=g)[:total]
    return out.view(w.batch, w.n_kv_heads, max(1, w.planted_groups), w.planted_blocks) \
              .permute(2, 0, 1, 3).contiguous()


def make_host_kv(w: Workload, layer: int = 0, device="cpu", out: torch.Tensor | None = None):
    """Full KV cache of one layer, bf16 [B, Hkv, N, 2, P, D].

    Keys and values ~ N(0,1) (keys Student-t(3) when ``key_dist`` says so),
    outlier channels scaled; planted blocks get keys
    ``planted_key_scale * u + noise`` with u the query mean direction of their
    group.  Generated one sequence at a time on ``device`` and written into
    ``out`` (for example a pinned host tensor) when given.
    """
    B, H, N, P, D = w.batch, w.n_kv_heads, w.max_blocks, w.block_tokens, w.head_dim
    if out is None:
        out = torch.empty(B, H, N, 2, P, D, dtype=torch.bfloat16, device=device)
    g = _gen(w, layer, _P_KV, device)
    cs = _channel_scale(w, layer, device).view(H, 1, 1, 1, D)
    plant = planted_positions(w, layer) if w.planted_blocks else None
    u = mean_directions(w, layer, device) if w.planted_blocks else None
    for b in range(B):
        keys = _draw_keys(w, (H, N, P, D), g, device) * cs.view(H, 1, 1, D)
        vals = torch.randn(H, N, P, D, generator=g, device=device) * cs.view(H, 1, 1, D)
        if plant is not None:
            for r in range(plant.shape[0]):
                for h in range(H):
                    ids = plant[r, b, h].to(device)
                    keys[h, ids] += w.planted_key_scale * u[r, b, h].view(1, 1, D)
        blk = torch.stack([keys, vals], dim=2).to(torch.bfloat16)   # [H, N, 2, P, D]
        out[b].copy_(blk)
    return out


def initial_ctx_len(w: Workload, device="cpu") -> torch.Tensor:
    return torch.full((w.batch,), w.context, dtype=torch.int32, device=device)


class QueryStream:
    """Per-step queries [B, Qn, Hq, D] bf16 for one layer.

    q[b, j, h*G+g] = m_t[b, h] + query_noise * xi with fresh xi per row.  The
    mean m_t = u + drift_scale * d_t: u is the per-(sequence, head) base
    direction (with planted groups, the direction of group
    (t // hop_every) mod groups) and d_t an AR(1) process
    d_t = rho * d_{t-1} + sqrt(1 - rho^2) * eta_t with unit stationary
    variance (absent when rho = 0).  Step 0 is the priming step (the drafts
    of the step before decoding starts).

    With ``draft_lead`` the drafts look ahead: row j of step t is drawn around
    m_{t+j}, the mean the verification row will have j steps later (the AR(1)
    path is generated that far ahead), so draft j stands for a draft model
    that proposes the token j positions on, whose query it carries (OasisKV
    Figure 6: the propagated draft query approximates the true next-token
    query).  Row 0 is drawn around m_t as before.  Without it every row of a
    step shares m_t.
    """

    def __init__(self, w: Workload, layer: int = 0, device="cpu"):
        self.w, self.layer, self.device = w, layer, device
        self.g = _gen(w, layer, _P_QUERY, device)
        self.u = mean_directions(w, layer, device)          # [groups, B, H, D]
        self.d = torch.randn(self.u.shape[1:], generator=self.g, device=device)
        self.t = 0
        if w.draft_lead:
            # d_t .. d_{t+Qn-1}: the drift of the verification row and of each draft's target step
            self.path = [self.d]
            for _ in range(w.n_queries - 1):
                self.path.append(self._ar_step(self.path[-1]))

    def _ar_step(self, d):
        eta = torch.randn(d.shape, generator=self.g, device=self.device)
        return self.w.ar_rho * d + math.sqrt(1.0 - self.w.ar_rho ** 2) * eta

    def _mean(self, t, d):
        w = self.w
        group = (t // w.hop_every) % self.u.shape[0] if w.hop_every else 0
        m = self.u[group]
        if w.ar_rho:
            m = m + (w.drift_scale * w.query_mean_scale) * d
        return m

    def next(self) -> torch.Tensor:
        w = self.w
        if w.draft_lead:
            return self._next_lead()
        group = (self.t // w.hop_every) % self.u.shape[0] if w.hop_every else 0
        m = self.u[group]
        if w.ar_rho:
            if self.t > 0:
                eta = torch.randn(self.d.shape, generator=self.g, device=self.device)
                self.d = w.ar_rho * self.d + math.sqrt(1.0 - w.ar_rho ** 2) * eta
            m = m + (w.drift_scale * w.query_mean_scale) * self.d
        B, H, G, D, Qn = w.batch, w.n_kv_heads, w.group, w.head_dim, w.n_queries
        xi = torch.randn(B, Qn, H, G, D, generator=self.g, device=self.device)
        q = m.view(B, 1, H, 1, D) + w.query_noise * xi
        self.t += 1
        return q.reshape(B, Qn, H * G, D).to(torch.bfloat16)

    def _next_lead(self) -> torch.Tensor:
        w = self.w
        B, H, G, D, Qn = w.batch, w.n_kv_heads, w.group, w.head_dim, w.n_queries
        means = torch.stack([self._mean(self.t + j, self.path[j]) for j in range(Qn)], dim=1)   # [B, Qn, H, D]
        xi = torch.randn(B, Qn, H, G, D, generator=self.g, device=self.device)
        q = means.view(B, Qn, H, 1, D) + w.query_noise * xi
        self.path = self.path[1:] + [self._ar_step(self.path[-1])]
        self.t += 1
        return q.reshape(B, Qn, H * G, D).to(torch.bfloat16)


def eviction_mask(w: Workload, layer: int, step: int, device="cpu") -> torch.Tensor:
    """Seeded Bernoulli(evict_prob) residency-loss mask, bool [B, Hkv, K]."""
    g = torch.Generator(device=device)
    g.manual_seed(w.seed + 100 * (_P_EVICT + 1) + 10007 * layer + 7919 * step)
    return torch.rand(w.batch, w.n_kv_heads, w.budget_blocks, generator=g, device=device) < w.evict_prob


def append_rows(w: Workload, layer: int, step: int, device="cpu"):
    """New token rows (k_new, v_new), bf16 [B, Hkv, D] each, for one step."""
    g = torch.Generator(device=device)
    g.manual_seed(w.seed + 100 * (_P_APPEND + 1) + 10007 * layer + 7919 * step)
    cs = _channel_scale(w, layer, device)
    k = _draw_keys(w, (w.batch, w.n_kv_heads, w.head_dim), g, device) * cs
    v = torch.randn(w.batch, w.n_kv_heads, w.head_dim, generator=g, device=device) * cs
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """Raw bf16 bit patterns of a tensor as a numpy uint16 array (CPU copy)."""
    import numpy as np
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
