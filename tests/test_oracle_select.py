"""Pins for the oracle's BF16 tile selection.

Planted tiles: Q and K tiles built from constant rows, so their pooled means
are known exactly and the tile scores are single products chosen by hand;
the selected tiles must be the planted ones.  The other pins are the
properties the rule fixes at any size: forced sink and diagonal tiles, the
top-k dominance of the chosen tiles, popcounts, causal emptiness, budget
extremes and nesting, and the hi-pair totals of the budget rule on the
measured workloads (closed-form counts that need no scores).
"""
import math

import numpy as np
import pytest
import torch

from mixed_precision_bit_quant_b200 import workloads
from oracle.select import (budget_for_row, mask_to_dense, pool_tiles, select,
                           select_rows, tile_scores)


def _bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _planted(T=8, d=64):
    """K tile j: every row = a_j * e_j; Q tile i: every row = sum_j b[i,j] e_j.

    score(i, j) = b[i,j] * a_j exactly (one non-zero product per pair)."""
    N = 128 * T
    a = np.array([2.0 ** (j % 3) for j in range(T)])          # 1, 2, 4, 1, 2, 4, ...
    b = np.zeros((T, T))
    for i in range(T):
        for j in range(T):
            b[i, j] = 0.0625 * ((3 * i + 5 * j) % 7 + 1)          # small distinct-ish values
        b[i, (i + 3) % T] = 32.0                                  # planted winners
        b[i, (i + 5) % T] = 16.0
    K = np.zeros((1, 1, N, d))
    Q = np.zeros((1, 1, N, d))
    for j in range(T):
        K[0, 0, j * 128:(j + 1) * 128, j] = a[j]
    for i in range(T):
        Q[0, 0, i * 128:(i + 1) * 128, :T] = b[i]
    return _bf16(Q), _bf16(K), a, b


def test_pooled_means_exact_for_constant_tiles():
    Q, K, a, b = _planted()
    qp = pool_tiles(Q)
    kp = pool_tiles(K)
    T = len(a)
    for j in range(T):
        want = np.zeros(64)
        want[j] = a[j]
        assert np.array_equal(kp[0, 0, j], want.astype(np.float32))
    for i in range(T):
        assert np.array_equal(qp[0, 0, i, :T], b[i].astype(np.float32))


def test_planted_tiles_are_selected():
    Q, K, a, b = _planted()
    T = len(a)
    res = select(Q, K, causal=False, budget_bp=0, budget_tiles=4)
    dense = mask_to_dense(res["mask"], T)[0, 0]
    for i in range(T):
        want = {0, i}
        # fill to 4 with the planted winners: scores b*a, the planted b's are far larger
        extra = sorted(((b[i, j] * a[j], -j, j) for j in range(T) if j not in want), reverse=True)
        for s, _, j in extra:
            if len(want) == 4:
                break
            want.add(j)
        assert set(np.nonzero(dense[i])[0].tolist()) == want, i
        # the planted pair is always among them unless forced already
        assert dense[i, (i + 3) % T]


def test_scores_are_products_of_planted_values():
    Q, K, a, b = _planted()
    sc = tile_scores(pool_tiles(Q), pool_tiles(K), 1, 1)[0, 0]
    assert np.array_equal(sc, (b * a[None, :]).astype(np.float32))


def _random_problem(seed=0, B=1, Hq=4, Hkv=2, N=1000, d=64):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, N, d), generator=g).to(torch.bfloat16)
    k = (torch.randn((B, Hkv, N, d), generator=g) + 0.5).to(torch.bfloat16)
    return q, k


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("bp,tiles", [(500, 0), (2500, 0), (0, 3), (9999, 0)])
def test_selection_invariants(causal, bp, tiles):
    q, k = _random_problem(seed=bp + tiles + int(causal))
    res = select(q, k, causal=causal, budget_bp=bp, budget_tiles=tiles)
    T = res["qp"].shape[2]
    dense = mask_to_dense(res["mask"], T)
    sc = res["scores"]
    B, H = dense.shape[:2]
    for b_ in range(B):
        for h in range(H):
            for i in range(T):
                n_i = i + 1 if causal else T
                row = dense[b_, h, i]
                assert not row[n_i:].any()                       # nothing outside C_i
                forced = {0, i} & set(range(n_i))
                k_i = budget_for_row(n_i, len(forced), bp, tiles)
                assert row.sum() == k_i == res["counts"][b_, h, i]
                if k_i == 0:
                    continue
                assert all(row[j] for j in forced)
                chosen = [j for j in range(n_i) if row[j] and j not in forced]
                others = [j for j in range(n_i) if not row[j]]
                for c in chosen:                                 # top-k dominance with index tie-break
                    for o in others:
                        sc_c, sc_o = float(sc[b_, h, i, c]), float(sc[b_, h, i, o])
                        assert sc_c > sc_o or (sc_c == sc_o and c < o)


def test_budget_extremes_and_nesting():
    q, k = _random_problem(seed=7, N=1500)
    T = 12
    full = mask_to_dense(select(q, k, True, 10000)["mask"], T)
    none = mask_to_dense(select(q, k, True, 0)["mask"], T)
    tri = np.tril(np.ones((T, T), dtype=bool))
    assert np.array_equal(full, np.broadcast_to(tri, full.shape))
    assert not none.any()
    prev = None
    for kk in range(1, T + 1):
        cur = mask_to_dense(select(q, k, False, 0, kk)["mask"], T)
        if prev is not None:
            assert np.all(cur >= prev)                           # budgets nest
        prev = cur


def _hi_total(w):
    T = w.T
    tot = pairs = 0
    for i in range(T):
        n_i = i + 1 if w.causal else T
        forced = len({0, i} & set(range(n_i)))
        tot += budget_for_row(n_i, forced, w.budget_bp, w.budget_tiles)
        pairs += n_i
    return tot * w.B * w.Hq, pairs * w.B * w.Hq


def test_hi_pair_totals_of_the_workloads():
    # totals of the budget rule, counted per head: BF16 pairs / all computed pairs
    W = workloads.WORKLOADS
    assert _hi_total(W["tiny"]) == (16, 32)
    assert _hi_total(W["vit"]) == (1152, 1536)
    assert _hi_total(W["llm8k"]) == (4960, 66560)
    assert _hi_total(W["llm32k"]) == (57184, 1052672)
    assert _hi_total(W["llm128k"]) == (855904, 16793600)


def test_ragged_pool_uses_valid_rows_only():
    x = np.zeros((1, 1, 197, 16), dtype=np.float32)
    x[0, 0, 128:, :] = 3.0
    x[0, 0, 128, 0] = 72.0                                       # 69 valid rows in the last tile
    p = pool_tiles(_bf16(x))
    assert p[0, 0, 1, 1] == 3.0
    assert p[0, 0, 1, 0] == np.float32((3.0 * 68 + 72.0) / 69.0)


def test_pooled_means_close_to_float64(rng):
    x = rng.standard_normal((1, 2, 300, 32)).astype(np.float32)
    xb = _bf16(x)
    p = pool_tiles(xb)
    xf = xb.double().numpy()
    for t in range(3):
        want = xf[:, :, t * 128:min(300, (t + 1) * 128)].mean(axis=2)
        assert np.allclose(p[:, :, t], want, rtol=1e-5, atol=1e-6)


def test_row_subset_matches_full_selection():
    q, k = _random_problem(seed=11, N=1200)
    full = select(q, k, True, 1500)
    rows = [(0, 0, 3), (0, 3, 9), (0, 1, 0)]
    part = select(q, k, True, 1500, rows=rows)
    for (b, h, i) in rows:
        assert np.array_equal(part["mask"][b, h, i], full["mask"][b, h, i])
        assert part["counts"][b, h, i] == full["counts"][b, h, i]
