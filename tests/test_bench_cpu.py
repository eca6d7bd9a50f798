"""The benchmark's host-side arithmetic (no GPU): the tile-pair counts behind the
roofline and the roofline's closed forms.

The pair counts must be the ones the selection rule produces, so they are
checked against the oracle's selection (mask popcounts on real selections of
the small workloads, and the oracle's per-row budget on the large ones); the
roofline is checked against what its definition fixes (all-FP4 and all-BF16
limits and their ratio under the nominal 4:2:1 rate ratios).
"""
import importlib.util
import os

import numpy as np
import pytest

from mixed_precision_bit_quant_b200 import workloads
from oracle import select as osel

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)


def _popcount(mask):
    return int(np.unpackbits(np.ascontiguousarray(mask).view(np.uint8)).sum())


@pytest.mark.parametrize("name", ["tiny", "vit"])
def test_pair_counts_equal_the_oracle_selection(name):
    w = workloads.WORKLOADS[name]
    q, k, _ = workloads.generate(w)
    sel = osel.select(q, k, w.causal, w.budget_bp, w.budget_tiles)
    hi, lo = bench.hi_lo_pairs(w)
    total = w.B * w.Hq * (w.T * (w.T + 1) // 2 if w.causal else w.T * w.T)
    assert hi == _popcount(sel["mask"]) == int(sel["counts"].sum())
    assert hi + lo == total


@pytest.mark.parametrize("name", ["llm8k", "llm32k", "llm128k"])
def test_pair_counts_equal_the_oracle_budget(name):
    w = workloads.WORKLOADS[name]
    hi = 0
    for i in range(w.T):
        n_i = i + 1
        hi += osel.budget_for_row(n_i, 1 if i == 0 else 2, w.budget_bp, w.budget_tiles)
    assert bench.hi_lo_pairs(w) == (hi * w.B * w.Hq, (w.T * (w.T + 1) // 2 - hi) * w.B * w.Hq)


def test_roofline_limits_and_ratio():
    peaks = {"bf16_tflops": 1000.0}
    w0 = workloads.WORKLOADS["llm8k"].with_budget(bp=0)
    w1 = workloads.WORKLOADS["llm8k"].with_budget(bp=10000)
    r0 = bench.attn_roofline(w0, peaks)
    r1 = bench.attn_roofline(w1, peaks)
    pairs = w0.B * w0.Hq * w0.T * (w0.T + 1) // 2
    F = 2.0 * 128 * 128 * w0.d
    assert r0["hi"] == 0 and r1["lo"] == 0 and r0["lo"] == r1["hi"] == pairs
    assert r0["flops"] == r1["flops"] == pairs * 2 * F
    # all BF16: both products at the BF16 rate; all FP4: QK^T at 4x, P.V at 2x
    assert r1["t_roof"] == pytest.approx(pairs * 2 * F / 1e15)
    assert r0["t_roof"] == pytest.approx(pairs * (F / 4e15 + F / 2e15))
    assert r1["t_roof"] / r0["t_roof"] == pytest.approx(8.0 / 3.0)
    assert r0["t_roof_fp4_both"] == pytest.approx(pairs * 2 * F / 4e15)


def test_roofline_of_the_32k_workload_with_the_measured_peak():
    peaks, kind = bench._peaks()
    r = bench.attn_roofline(workloads.WORKLOADS["llm32k"], peaks)
    assert (r["hi"], r["lo"]) == (57184, 1052672 - 57184)
    if kind == "measured":
        assert r["t_roof"] == pytest.approx(2.19e-3, rel=5e-3)
