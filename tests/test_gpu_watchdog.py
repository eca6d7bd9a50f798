"""Device watchdog: a bounded wait that runs out ends the kernel with a status, not a hang.

The test withholds one V copy through the library's test hook, so the P.V
issuer waits for a barrier that nothing will complete.  The wait gives up
after its limit, the work tile raises the abort flag, every role returns
(copies in flight drained, tensor memory released), and the host reads
THRIFT_ERR_TIMEOUT.  A normal call afterwards must run clean and reproduce
the output of a call made before the fault, so the context stayed usable.
"""
import time

import pytest
import torch

import mixed_precision_bit_quant_b200 as mq
from mixed_precision_bit_quant_b200 import _lib, workloads

pytestmark = pytest.mark.gpu


def _problem():
    w = workloads.custom("watchdog", 1, 1, 1, 256, 128, False, "llm", 0, 0, seed=5)  # 2 tiles, all FP4
    q, k, v = (t.cuda() for t in workloads.generate(w))
    return w, q, k, v


def test_withheld_copy_times_out_and_context_survives():
    w, q, k, v = _problem()
    quant = mq.quantize(q, k, v, w.causal)
    mask, _ = mq.select(q, k, w.causal, w.budget_bp, w.budget_tiles)
    o_ref, _ = mq.attn_fwd(q, k, quant, mask, w.causal)
    assert mq.device_status() == (0, 0)

    mq.debug_withhold_v_load(1)
    try:
        t0 = time.time()
        o_bad, _ = mq.attn_fwd(q, k, quant, mask, w.causal)
        status, word = mq.device_status()
        elapsed = time.time() - t0
    finally:
        mq.debug_withhold_v_load(-1)
    assert status == _lib.THRIFT_ERR_TIMEOUT, (status, hex(word))
    assert word & 2, hex(word)                 # raised by an issuer's wait
    assert 1.5 < elapsed < 30.0, elapsed       # the 2 s limit, not an endless spin
    del o_bad                                  # undefined by contract

    o_again, _ = mq.attn_fwd(q, k, quant, mask, w.causal)
    assert mq.device_status() == (0, 0)
    assert torch.equal(o_again.view(torch.int16), o_ref.view(torch.int16))
