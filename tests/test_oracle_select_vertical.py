"""Pins of the vertical-line selection mode (oracle/select.py, select_rows_vertical).

The votes are checked against the score mode's own masks (pinned separately
in test_oracle_select.py), the fill against the ordering the mode defines
(every chosen tile ranks above every candidate left out), and a planted
vertical line against the outcome the definition implies.
"""
import numpy as np
import pytest

from mixed_precision_bit_quant_b200 import workloads
from oracle import select as osel


def _dense(mask, T):
    return osel.mask_to_dense(mask, T)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("bp,bt", [(2500, 0), (4000, 0), (0, 4), (0, 1)])
def test_votes_fill_and_counts_by_brute_force(causal, bp, bt):
    rng = np.random.default_rng(11)
    B, H, T = 2, 3, 12
    sc = rng.standard_normal((B, H, T, T)).astype(np.float32)
    sc[0, 0, :, 5] = sc[0, 0, :, 6]                       # exact score ties across columns
    m_s, c_s = osel.select_rows(sc, causal, bp, bt)
    m_v, c_v, votes = osel.select_rows_vertical(sc, causal, bp, bt)
    assert np.array_equal(c_s, c_v)                        # same budget per row
    ds, dv = _dense(m_s, T), _dense(m_v, T)
    for b in range(B):
        for h in range(H):
            want_votes = np.zeros(T, np.int64)
            for i in range(T):
                forced = {0, i} & set(range(i + 1 if causal else T))
                for j in np.nonzero(ds[b, h, i])[0]:
                    if j not in forced:
                        want_votes[j] += 1
            assert np.array_equal(votes[b, h], want_votes)
            for i in range(T):
                n_i = i + 1 if causal else T
                forced = {0, i} & set(range(n_i))
                chosen = set(np.nonzero(dv[b, h, i])[0])
                if c_v[b, h, i] == 0:
                    assert not chosen
                    continue
                assert forced <= chosen and max(chosen) < n_i
                key = lambda j: (votes[b, h, j], float(sc[b, h, i, j]), -j)   # noqa: E731
                picked = [key(j) for j in chosen - forced]
                left = [key(j) for j in set(range(n_i)) - chosen]
                if picked and left:
                    assert min(picked) > max(left)


def test_planted_vertical_line_is_taken_by_every_row():
    # a key tile that sits near the top of every row collects the most votes; by the
    # definition it then ranks first for every row that has budget to fill and sees
    # it as a non-forced candidate, even rows whose own scores put it third or lower
    rng = np.random.default_rng(12)
    T, js = 40, 17
    sc = rng.uniform(-1.0, 1.0, (1, 1, T, T)).astype(np.float32)
    sc[0, 0, :, js] = 0.9 + 0.05 * rng.uniform(size=T).astype(np.float32)
    m_v, c_v, votes = osel.select_rows_vertical(sc, False, 0, 5)   # 2 forced + 3 filled
    v = votes[0, 0]
    assert v[js] > np.delete(v, js).max()
    dv = _dense(m_v, T)[0, 0]
    assert dv[:, js].all()
    m_s, _ = osel.select_rows(sc, False, 0, 5)
    ds = _dense(m_s, T)[0, 0]
    assert not ds[:, js].all()                       # the score mode leaves it out of some rows


@pytest.mark.parametrize("causal", [False, True])
def test_degenerate_budgets_match_the_score_mode(causal):
    w = workloads.custom("v", 1, 2, 1, 1500, 64, causal, "llm", 500, 0, seed=4)
    q, k, _ = workloads.generate(w)
    for bp, bt in ((0, 0), (10000, 0), (0, 2)):
        a = osel.select(q, k, causal, bp, bt)
        b = osel.select_vertical(q, k, causal, bp, bt)
        assert np.array_equal(a["mask"], b["mask"]) and np.array_equal(a["counts"], b["counts"])
    assert not osel.select_vertical(q, k, causal, 0, 0)["votes"].any()


def test_single_tile_problem():
    sc = np.zeros((1, 1, 1, 1), np.float32)
    m, c, v = osel.select_rows_vertical(sc, True, 500, 0)
    assert c[0, 0, 0] == 1 and m[0, 0, 0, 0] == 1 and v.sum() == 0
