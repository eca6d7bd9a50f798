"""Fixtures under tests/golden/.

thrift_abstract_budget.txt holds the one number the pages print for the
method itself (ThriftAttention: Selective Mixed Precision for Long-Context FP4
Attention, Abstract: 5% of the query-key blocks in high precision); the tests
check that it is the library's default budget and what the selection rule
turns it into.  oracle_snapshot.txt is a regression snapshot of the oracle's
integer outputs, written by tests/golden/make_oracle_snapshot.py from the
oracle alone.
"""
import importlib.util
import inspect
import math
import os

import mixed_precision_bit_quant_b200 as mq
from mixed_precision_bit_quant_b200 import workloads
from oracle import select as osel

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _fixture(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, value = line.split(None, 1)
                out[key] = value
    return out


def test_page_budget_is_the_default_budget():
    pct = int(_fixture("thrift_abstract_budget.txt")["high_precision_block_percent"])
    bp = pct * 100  # basis points of the candidate tiles
    assert inspect.signature(mq.select).parameters["budget_bp"].default == bp
    assert inspect.signature(mq.attention).parameters["budget_bp"].default == bp
    for name in ("llm8k", "llm32k", "llm128k"):
        assert workloads.WORKLOADS[name].budget_bp == bp


def test_page_budget_through_the_selection_rule():
    # a query tile with n candidates keeps ceil(5% of n) tiles, but never fewer than
    # its forced sink and diagonal tiles, so the share is at least the page's 5%
    pct = int(_fixture("thrift_abstract_budget.txt")["high_precision_block_percent"])
    for n in range(1, 1025):
        forced = 1 if n == 1 else 2
        k = osel.budget_for_row(n, forced, pct * 100, 0)
        assert k == min(n, max(forced, math.ceil(pct * n / 100)))
        assert k >= pct * n / 100
    # long rows: the forced tiles no longer matter and the share tends to 5%
    assert osel.budget_for_row(256, 2, pct * 100, 0) == 13


def test_oracle_snapshot_unchanged():
    spec = importlib.util.spec_from_file_location("make_oracle_snapshot",
                                                  os.path.join(GOLDEN, "make_oracle_snapshot.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    with open(os.path.join(GOLDEN, "oracle_snapshot.txt")) as f:
        stored = [line.strip() for line in f if line.strip() and not line.startswith("#")]
    assert mod.snapshot_lines() == stored


def _rational(expr: str):
    from fractions import Fraction
    out = Fraction(1)
    for factor in expr.split("*"):
        parts = factor.split("/")
        f = Fraction(int(parts[0]))
        for p in parts[1:]:
            f /= int(p)
        out *= f
    return out


def p_cast_problem(e_t: float):
    """The two-key problem of p_cast_closed_forms.txt: logits (0, -t) on row 0."""
    import torch
    d, N = 64, 2
    q = torch.zeros((1, 1, N, d), dtype=torch.float32)
    k = torch.zeros((1, 1, N, d), dtype=torch.float32)
    v = torch.zeros((1, 1, N, d), dtype=torch.float32)
    q[0, 0, 0, 0] = 10.5
    k[0, 0, 1, 0] = -10.5
    v[0, 0, 0, 0] = 1.0
    v[0, 0, 1, 1] = 1.0
    scale = math.log(e_t) / 110.25
    return tuple(t.to(torch.bfloat16) for t in (q, k, v)) + (scale,)


def p_cast_cases():
    cases = []
    with open(os.path.join(GOLDEN, "p_cast_closed_forms.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                name, tile, e_t, o0, o1 = line.split()
                cases.append((name, tile, float(e_t), _rational(o0), _rational(o1)))
    return cases


def test_p_cast_closed_forms():
    import numpy as np
    from oracle.attention import attn_forward
    from oracle.quantize import quantize
    cases = p_cast_cases()
    assert [c[0] for c in cases] == ["A", "B", "C", "D"]
    for name, tile, e_t, o0, o1 in cases:
        q, k, v, scale = p_cast_problem(e_t)
        qz = quantize(q, k, v)
        # the operands are exact in both precisions: only the cast of P rounds
        assert int(qz["q_sf"][0, 0, 0, 0]) == 0x7E and float(qz["q_g"][0, 0]) == 2.0 ** -8
        mask = np.full((1, 1, 1, 1), 1 if tile == "bf16" else 0, dtype=np.uint32)
        O, lse = attn_forward(q, k, v, qz, mask, False, sm_scale=scale)
        assert abs(O[0, 0, 0, 0] - float(o0)) <= 1e-12 * float(o0), name
        assert abs(O[0, 0, 0, 1] - float(o1)) <= 1e-12 * float(o1), name
        assert not O[0, 0, 0, 2:].any()
        assert np.allclose(O[0, 0, 1, :2], 0.5, rtol=0, atol=1e-15) and not O[0, 0, 1, 2:].any()
        assert abs(lse[0, 0, 0] - math.log(1.0 + 1.0 / e_t)) < 1e-12
