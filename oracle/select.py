"""Oracle: choosing the query-key tile pairs that run in BF16.

TEST INFRASTRUCTURE (see ``oracle/formats.py``): only tests, the smoke check
and the benchmark's CPU-baseline leg use this module.

What it follows.  ThriftAttention: Selective Mixed Precision for
Long-Context FP4 Attention (abstract, first stage): a cheap heuristic picks
a small number of important query-key block pairs for high precision.
HyQuant: Hybrid-Precision Quantization for LLM Attention (abstract) keeps
vertical-line (sink) tokens and the local window in high precision.  The
pages do not give the heuristic, so this library fixes it:

1. pool: per 128-row tile t and channel c, the mean of the original BF16
   values over the tile's valid rows, summed in FP32 in ascending row order
   and divided by the row count;
2. score(i, j) = sum_c qp[h][i][c] * kp[h/G][j][c], FP32 products and FP32
   additions in ascending c, starting from +0 (no fused multiply-add);
3. candidates C_i = {0..i} (causal) or {0..T-1}; forced F_i = {0, i} & C_i
   (sink tile and diagonal / local window);
4. budget k_i: ``budget_tiles > 0`` -> min(n_i, max(|F_i|, budget_tiles));
   else bp = budget_bp: 0 -> 0 (no forced tiles either), >= 10000 -> n_i,
   otherwise min(n_i, max(|F_i|, ceil(bp * n_i / 10000)));
5. the forced tiles (when k_i > 0) plus the k_i - |F_i| best remaining
   candidates by (score descending, index ascending; -0 equals +0).

The result is a bitmask ``mask[B,Hq,T,ceil(T/32)]`` of uint32 words: bit
j % 32 of word j // 32 set means tile pair (i, j) runs in BF16.

Parity pins: tests/test_oracle_select.py (planted scores recover the planted
tiles, top-k dominance, popcounts, causal emptiness, budget extremes,
nesting of budgets, pooled means against float64 means).

A second mode, ``select_vertical``, ranks the fill by column votes (HyQuant's
vertical lines); its definition is in ``select_rows_vertical`` and its pins in
tests/test_oracle_select_vertical.py.
"""
from __future__ import annotations

import numpy as np
import torch

F32 = np.float32


def _as_f32(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float32).numpy()
    return np.asarray(x, dtype=np.float32)


def pool_tiles(x) -> np.ndarray:
    """x[B,H,N,d] -> per-tile column means [B,H,T,d] (FP32, ascending row sums)."""
    x = _as_f32(x)
    B, H, N, d = x.shape
    T = (N + 127) // 128
    out = np.zeros((B, H, T, d), dtype=F32)
    for t in range(T):
        r0 = t * 128
        cnt = min(128, N - r0)
        acc = np.zeros((B, H, d), dtype=F32)
        for r in range(cnt):
            acc = (acc + x[:, :, r0 + r, :]).astype(F32)
        out[:, :, t, :] = (acc / F32(cnt)).astype(F32)
    return out


def tile_scores(qp, kp, Hq: int, Hkv: int) -> np.ndarray:
    """scores[B,Hq,T,T] = FP32 dot products of pooled means, ascending c."""
    qp = np.asarray(qp, dtype=F32)
    kp = np.asarray(kp, dtype=F32)
    G = Hq // Hkv
    kp_q = np.repeat(kp, G, axis=1)                  # query head h uses kv head h // G
    B, H, T, d = qp.shape
    acc = np.zeros((B, H, T, T), dtype=F32)
    for c in range(d):
        prod = (qp[:, :, :, None, c] * kp_q[:, :, None, :, c]).astype(F32)
        acc = (acc + prod).astype(F32)
    return acc


def budget_for_row(n_i: int, n_forced: int, budget_bp: int, budget_tiles: int) -> int:
    if budget_tiles > 0:
        return min(n_i, max(n_forced, budget_tiles))
    if budget_bp <= 0:
        return 0
    if budget_bp >= 10000:
        return n_i
    want = (budget_bp * n_i + 9999) // 10000
    return min(n_i, max(n_forced, want))


def select_rows(scores, causal: bool, budget_bp: int, budget_tiles: int, rows=None):
    """scores[B,Hq,T,T] -> (mask[B,Hq,T,W] uint32, counts[B,Hq,T] int32).

    ``rows``: optional list of (b, h, i) query tiles to fill (others stay 0).
    """
    scores = np.asarray(scores, dtype=F32)
    B, H, T, _ = scores.shape
    W = (T + 31) // 32
    mask = np.zeros((B, H, T, W), dtype=np.uint32)
    counts = np.zeros((B, H, T), dtype=np.int32)
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(H) for i in range(T)]
    for (b, h, i) in rows:
        n_i = i + 1 if causal else T
        forced = sorted({0, i} & set(range(n_i)))
        k_i = budget_for_row(n_i, len(forced), budget_bp, budget_tiles)
        chosen = []
        if k_i > 0:
            chosen = list(forced)
            rest = [j for j in range(n_i) if j not in forced]
            s = scores[b, h, i, rest].astype(np.float64)   # -0 == +0 in comparisons
            order = np.lexsort((np.asarray(rest), -s))     # score desc, then index asc
            chosen += [rest[o] for o in order[: k_i - len(forced)]]
        for j in chosen:
            mask[b, h, i, j // 32] |= np.uint32(1) << np.uint32(j % 32)
        counts[b, h, i] = len(chosen)
    return mask, counts


def select(q, k, causal: bool, budget_bp: int, budget_tiles: int = 0, rows=None):
    """The library's ``thrift_select``: pooled scores -> BF16 tile mask.

    ``rows``: optional list of (b, h, i) query tiles to compute (others stay 0).
    """
    qp = pool_tiles(q)
    kp = pool_tiles(k)
    Hq, Hkv = qp.shape[1], kp.shape[1]
    if rows is None:
        sc = tile_scores(qp, kp, Hq, Hkv)
    else:
        # scores only for the requested query tiles (same products and order)
        B, _, T, d = qp.shape
        sc = np.zeros((B, Hq, T, T), dtype=F32)
        G = Hq // Hkv
        for (b, h, i) in rows:
            sc[b, h, i] = tile_scores(qp[b:b + 1, h:h + 1, i:i + 1], kp[b:b + 1, h // G:h // G + 1], 1, 1)[0, 0, 0]
    mask, counts = select_rows(sc, causal, budget_bp, budget_tiles, rows)
    return dict(qp=qp, kp=kp, scores=sc, mask=mask, counts=counts)


def select_rows_vertical(scores, causal: bool, budget_bp: int, budget_tiles: int):
    """The vertical-line selection mode: scores[B,Hq,T,T] -> (mask, counts, votes).

    HyQuant: Hybrid-Precision Quantization for LLM Attention (abstract) keeps
    "vertical-line" tokens -- keys that many queries attend to -- and the local
    window in high precision, chosen by a lightweight attention-pattern signal;
    the page gives no formula, so this library fixes one at tile level, in
    integers so that it is exactly reproducible:

    1. every query tile i of a (batch, head) votes for the tiles the score mode
       would add to its forced ones: its k_i - |F_i| best non-forced candidates
       by (score desc, index asc);
    2. votes[b, h, j] = the number of query tiles of (b, h) voting for key tile j
       (the column-importance signal);
    3. each query tile keeps its forced tiles (sink 0 and diagonal i) and fills
       its budget with the non-forced candidates ranked by (votes desc, score
       desc, index asc).

    The budget k_i and the forced set are those of the score mode, so every row
    keeps the same number of BF16 tiles in both modes.
    """
    scores = np.asarray(scores, dtype=F32)
    B, H, T, _ = scores.shape
    W = (T + 31) // 32
    votes = np.zeros((B, H, T), dtype=np.int64)
    plan = []
    for b in range(B):
        for h in range(H):
            for i in range(T):
                n_i = i + 1 if causal else T
                forced = sorted({0, i} & set(range(n_i)))
                k_i = budget_for_row(n_i, len(forced), budget_bp, budget_tiles)
                rest = [j for j in range(n_i) if j not in forced]
                fill = max(0, k_i - len(forced)) if k_i > 0 else 0
                s = scores[b, h, i, rest].astype(np.float64)
                by_score = [rest[o] for o in np.lexsort((np.asarray(rest), -s))]
                for j in by_score[:fill]:
                    votes[b, h, j] += 1
                plan.append((b, h, i, k_i, forced, rest, fill))
    mask = np.zeros((B, H, T, W), dtype=np.uint32)
    counts = np.zeros((B, H, T), dtype=np.int32)
    for (b, h, i, k_i, forced, rest, fill) in plan:
        chosen = []
        if k_i > 0:
            chosen = list(forced)
            s = scores[b, h, i, rest].astype(np.float64)
            v = votes[b, h, rest].astype(np.float64)
            order = np.lexsort((np.asarray(rest), -s, -v))   # votes desc, score desc, index asc
            chosen += [rest[o] for o in order[:fill]]
        for j in chosen:
            mask[b, h, i, j // 32] |= np.uint32(1) << np.uint32(j % 32)
        counts[b, h, i] = len(chosen)
    return mask, counts, votes


def select_vertical(q, k, causal: bool, budget_bp: int, budget_tiles: int = 0):
    """Pooled scores -> BF16 tile mask in the vertical-line mode (see select_rows_vertical)."""
    qp = pool_tiles(q)
    kp = pool_tiles(k)
    sc = tile_scores(qp, kp, qp.shape[1], kp.shape[1])
    mask, counts, votes = select_rows_vertical(sc, causal, budget_bp, budget_tiles)
    return dict(qp=qp, kp=kp, scores=sc, mask=mask, counts=counts, votes=votes)


def mask_bit(mask, b: int, h: int, i: int, j: int) -> bool:
    return bool((int(mask[b, h, i, j // 32]) >> (j % 32)) & 1)


def mask_to_dense(mask, T: int) -> np.ndarray:
    """[B,H,T,W] words -> [B,H,T,T] bool."""
    m = np.asarray(mask, dtype=np.uint32)
    B, H, Tq, W = m.shape
    bits = ((m[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool)
    return bits.reshape(B, H, Tq, W * 32)[..., :T]
