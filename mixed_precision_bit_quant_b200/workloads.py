"""Seeded synthetic workloads for the mixed FP4/BF16 attention forward.

This module only draws random numbers.  It holds none of the method's
arithmetic (no quantisation, no selection, no attention), so that both the
CUDA path and the CPU oracle can be fed the very same bytes without sharing
any code that computes a result.

Every workload is a set of BF16 tensors ``q[B,Hq,N,d]``, ``k[B,Hkv,N,d]`` and
``v[B,Hkv,N,d]`` (contiguous, head-major) drawn on the host with
``torch.Generator().manual_seed(seed)`` in the fixed order Q, K, structure
(offsets / outlier channels), V.  The shapes follow the workloads the pages
study: long-context LLM prefill with grouped-query heads (ThriftAttention:
Selective Mixed Precision for Long-Context FP4 Attention, abstract: the gain
"grows with sequence length"), attention sinks / vertical lines and local
windows (HyQuant: Hybrid-Precision Quantization for LLM Attention, abstract),
and ViT-shaped attention (QFlash, abstract: ViT/DeiT/Swin workloads).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    kind: str                 # "tiny" | "vit" | "llm"
    budget_bp: int = 500      # BF16 budget in basis points of candidate tiles
    budget_tiles: int = 0     # >0 overrides budget_bp with a tile count per query tile
    seed: int = 0

    @property
    def T(self) -> int:
        return (self.N + 127) // 128

    def with_budget(self, bp: Optional[int] = None, tiles: Optional[int] = None) -> "Workload":
        return dataclasses.replace(
            self,
            budget_bp=self.budget_bp if bp is None else bp,
            budget_tiles=self.budget_tiles if tiles is None else tiles,
        )

    def causal_adjusted_flops(self) -> float:
        """Effective attention FLOPs: 4*B*Hq*N^2*d, halved for causal runs."""
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.d
        return f / 2.0 if self.causal else f


# The five workloads the library is measured and checked on.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 2, 512, 64, False, "tiny", budget_bp=0, budget_tiles=2, seed=0),
    "vit": Workload("vit", 32, 12, 12, 197, 64, False, "vit", budget_bp=500, seed=0),
    "llm8k": Workload("llm8k", 1, 32, 8, 8192, 128, True, "llm", budget_bp=500, seed=0),
    "llm32k": Workload("llm32k", 1, 32, 8, 32768, 128, True, "llm", budget_bp=500, seed=0),
    "llm128k": Workload("llm128k", 1, 32, 8, 131072, 128, True, "llm", budget_bp=500, seed=0),
}

# A quality-axis workload with attention structure away from the sink: the
# llm8k draw plus planted vertical lines (HyQuant: Hybrid-Precision
# Quantization for LLM Attention, abstract: "vertical-line" tokens that many
# queries attend to).  Not a benchmark configuration.
VLINES = Workload("llm8k_vlines", 1, 32, 8, 8192, 128, True, "llm_vlines", budget_bp=500, seed=0)


def custom(name: str, B: int, Hq: int, Hkv: int, N: int, d: int, causal: bool,
           kind: str = "llm", budget_bp: int = 500, budget_tiles: int = 0, seed: int = 0) -> Workload:
    return Workload(name, B, Hq, Hkv, N, d, causal, kind, budget_bp, budget_tiles, seed)


def generate(w: Workload, device: str = "cpu"):
    """Draw (q, k, v) as BF16 tensors for workload ``w``.

    tiny: Q, V ~ N(0,1); K = N(0,1) + 4*u with u ~ N(0,1) per (head, channel);
          key 0 of every head scaled by 8 (an attention sink).
    vit:  Q, K, V ~ N(0,1); one shared set of max(1, round(0.02*d)) outlier
          channels, drawn once, scaled by 10 in Q, K and V.
    llm:  Q, K ~ N(0,1); a per-(kv head, channel) offset ~ N(0, std 2) added
          to every key; key 0 scaled by 8 (sink); V ~ N(0,1).
    llm_vlines: the llm draw, then per (batch, kv head) a direction u ~ N(0,1)^d:
          16 random keys in each of 3 random key tiles (not tile 0) get + 2u and
          every query of the group + 0.25u (planted vertical lines).
    """
    g = torch.Generator().manual_seed(w.seed)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    q = torch.randn((B, Hq, N, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32)
    if w.kind == "tiny":
        u = torch.randn((B, Hkv, 1, d), generator=g, dtype=torch.float32)
        k = k + 4.0 * u
        k[:, :, 0, :] *= 8.0
        v = torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32)
    elif w.kind == "vit":
        n_out = max(1, int(round(0.02 * d)))
        chans = torch.randperm(d, generator=g)[:n_out]
        v = torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32)
        for t in (q, k, v):
            t[..., chans] *= 10.0
    elif w.kind in ("llm", "llm_vlines"):
        off = 2.0 * torch.randn((B, Hkv, 1, d), generator=g, dtype=torch.float32)
        k = k + off
        k[:, :, 0, :] *= 8.0
        v = torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32)
        if w.kind == "llm_vlines":
            # per (batch, kv head): a direction u ~ N(0, 1)^d, 16 keys in each of 3 key
            # tiles (never tile 0) get + 2 u, and every query of the group + 0.25 u, so those
            # keys stand out for all queries (logit lift 0.5 |u|^2 / sqrt(d) ~ 0.5 sqrt(d))
            T = (N + 127) // 128
            G = Hq // Hkv
            for b in range(B):
                for hk in range(Hkv):
                    u = torch.randn((d,), generator=g, dtype=torch.float32)
                    tiles = 1 + torch.randperm(max(1, T - 1), generator=g)[:min(3, T - 1)]
                    for t in tiles.tolist():
                        cnt = min(128, N - 128 * t)
                        rows = 128 * t + torch.randperm(cnt, generator=g)[:min(16, cnt)]
                        k[b, hk, rows] += 2.0 * u
                    q[b, G * hk:G * (hk + 1)] += 0.25 * u
    else:
        raise ValueError(f"unknown workload kind {w.kind!r}")
    out = tuple(t.to(torch.bfloat16).contiguous() for t in (q, k, v))
    if device != "cpu":
        out = tuple(t.to(device) for t in out)
    return out


def sample_query_tiles(w: Workload, count: int = 64, seed: int = 1):
    """A fixed sample of (b, hq, query tile) triples, drawn with ``seed``."""
    g = torch.Generator().manual_seed(seed)
    total = w.B * w.Hq * w.T
    count = min(count, total)
    idx = torch.randperm(total, generator=g)[:count].tolist()
    out = []
    for f in sorted(idx):
        b, rem = divmod(f, w.Hq * w.T)
        h, i = divmod(rem, w.T)
        out.append((b, h, i))
    return out
