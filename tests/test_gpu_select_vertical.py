"""GPU parity of the vertical-line selection mode (thrift_select_vertical).

Masks and counts must equal the oracle's ``select_vertical`` bit for bit on
every workload (HyQuant: Hybrid-Precision Quantization for LLM Attention,
abstract: vertical-line keys and the local window in high precision; the
vote rule is this library's reading, stated in oracle/select.py).  The
attention kernel takes any mask, so one end-to-end case checks the output of
a vertically selected mask against the oracle as well.
"""
import numpy as np
import pytest

import mixed_precision_bit_quant_b200 as mq
from mixed_precision_bit_quant_b200 import workloads
from oracle import attention as oatt
from oracle import select as osel

pytestmark = pytest.mark.gpu


def _run(q, k, causal, bp, bt):
    qd, kd = q.cuda(), k.cuda()
    mask, counts = mq.select(qd, kd, causal, bp, bt, mode="vertical")
    st, word = mq.device_status()
    assert st == 0, f"device watchdog raised {word:#x}"
    ref = osel.select_vertical(q, k, causal, bp, bt)
    assert np.array_equal(mask.cpu().numpy().view(np.uint32), ref["mask"]), "vertical mask"
    assert np.array_equal(counts.cpu().numpy(), ref["counts"]), "vertical counts"
    return ref


@pytest.mark.parametrize("name", ["tiny", "vit", "llm8k", "llm32k", "llm128k"])
def test_vertical_masks_on_workloads(name):
    w = workloads.WORKLOADS[name]
    q, k, _ = workloads.generate(w)
    ref = _run(q, k, w.causal, w.budget_bp, w.budget_tiles)
    if name in ("llm8k", "llm32k"):
        # the vote signal must move some tiles, or this test would only repeat the score mode
        score = osel.select_rows(ref["scores"], w.causal, w.budget_bp, w.budget_tiles)[0]
        assert not np.array_equal(score, ref["mask"])


@pytest.mark.parametrize("N,Hq,Hkv,causal,bp,bt", [
    (1, 2, 1, True, 500, 0),
    (300, 4, 2, False, 2500, 0),
    (1000, 4, 4, True, 3000, 0),
    (1536, 2, 1, False, 0, 4),
    (640, 8, 2, True, 10000, 0),
    (640, 8, 2, True, 0, 0),
])
def test_vertical_shapes_and_budgets(N, Hq, Hkv, causal, bp, bt):
    w = workloads.custom("vcase", 1, Hq, Hkv, N, 64 if N % 2 else 128, causal, "llm", bp, bt, seed=N)
    q, k, _ = workloads.generate(w)
    _run(q, k, causal, bp, bt)


def test_vertical_mask_through_attention():
    w = workloads.custom("vattn", 1, 4, 2, 1100, 128, True, "llm", 2500, 0, seed=21)
    q, k, v = workloads.generate(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, _ = mq.attention(qd, kd, vd, True, 2500, mode="vertical")
    st, word = mq.device_status()
    assert st == 0, f"device watchdog raised {word:#x}"
    ref = osel.select_vertical(q, k, True, 2500)
    O_ref, _ = oatt.attn_forward(q, k, v, None, ref["mask"], True)
    og = o.float().cpu().numpy().astype(np.float64)
    err = np.abs(og - O_ref).max() / np.abs(O_ref).max()
    rel = np.linalg.norm(og - O_ref) / np.linalg.norm(O_ref)
    assert err <= 2e-2 and rel <= 5e-3, (err, rel)
