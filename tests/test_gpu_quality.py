"""Quality axis: error of the GPU output against exact FP64 softmax attention.

ThriftAttention: Selective Mixed Precision for Long-Context FP4 Attention
(abstract) claims that keeping about 5% of the query-key blocks in high
precision recovers most of the gap between FP4 and FP16 attention, because
the quantisation error concentrates on a few important interactions.  This
file measures that axis for the library's output: relative L2 and max error
of ``thrift_attn_fwd`` (through the C ABI) against textbook attention on the
BF16 inputs, at 0%, 5% and 100% BF16 budget, plus two controls at the 5%
budget: the same number of BF16 tiles per query tile picked at random
(forced sink and diagonal kept), and the forced tiles alone; and the
vertical-line selection mode at the same budget.  Besides the benchmark
workloads, a llm8k draw with planted vertical lines (workloads.VLINES) puts
attention structure away from the sink, where the selection has to find it.

"Gap recovered" = (e_0 - e_5) / (e_0 - e_100) on the relative L2 error.

The numbers are reported, not gated (beyond sanity: all-BF16 beats all-FP4).
With THRIFT_QUALITY_OUT set, the table is written there as JSON.
"""
import json
import os

import numpy as np
import pytest
import torch

import mixed_precision_bit_quant_b200 as mq
from mixed_precision_bit_quant_b200 import workloads
from oracle.attention import exact_attention_tiles

pytestmark = pytest.mark.gpu

_RESULTS = {}


def _random_mask(counts: np.ndarray, causal: bool, T: int, seed: int) -> np.ndarray:
    """A mask with counts[b,h,i] BF16 tiles per query tile: forced {0, i} plus random others."""
    rng = np.random.default_rng(seed)
    B, H, _ = counts.shape
    W = (T + 31) // 32
    m = np.zeros((B, H, T, W), dtype=np.uint32)
    for b in range(B):
        for h in range(H):
            for i in range(T):
                k = int(counts[b, h, i])
                if k == 0:
                    continue
                n = i + 1 if causal else T
                forced = [0] if i == 0 else [0, i]
                forced = [j for j in forced if j < n]
                others = np.array([j for j in range(n) if j not in forced], dtype=np.int64)
                pick = list(forced) + list(rng.choice(others, size=max(0, k - len(forced)), replace=False))
                for j in pick:
                    m[b, h, i, j // 32] |= np.uint32(1) << np.uint32(j % 32)
    return m


def _forced_mask(counts: np.ndarray, causal: bool, T: int) -> np.ndarray:
    B, H, _ = counts.shape
    W = (T + 31) // 32
    m = np.zeros((B, H, T, W), dtype=np.uint32)
    for i in range(T):
        for j in ([0] if i == 0 else [0, i]):
            m[:, :, i, j // 32] |= np.uint32(1) << np.uint32(j % 32)
    return m


def _err(o: torch.Tensor, ref: np.ndarray, sel):
    og = o.float().cpu().numpy().astype(np.float64)[sel]
    r = ref[sel]
    return {"rel_l2": float(np.linalg.norm(og - r) / np.linalg.norm(r)),
            "max_rel": float(np.abs(og - r).max() / np.abs(r).max())}


def _quality(w, tiles=None):
    q, k, v = workloads.generate(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    quant = mq.quantize(qd, kd, vd)
    T = w.T
    if tiles is None:
        tiles = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(T)]
    ref = exact_attention_tiles(q, k, v, w.causal, tiles)
    sel = ~np.isnan(ref[..., 0])
    out = {}
    for bp in (0, 500, 10000):
        mask, counts = mq.select(qd, kd, w.causal, bp)
        o, _ = mq.attn_fwd(qd, kd, quant, mask, w.causal)
        out[f"bp{bp}"] = _err(o, ref, sel)
        if bp == 500:
            mv, _ = mq.select(qd, kd, w.causal, bp, mode="vertical")
            o3, _ = mq.attn_fwd(qd, kd, quant, mv, w.causal)
            out["bp500_vertical_mode"] = _err(o3, ref, sel)
            cnt = counts.cpu().numpy()
            for name, m in (("bp500_random", _random_mask(cnt, w.causal, T, seed=7)),
                            ("forced_only", _forced_mask(cnt, w.causal, T))):
                md = torch.from_numpy(m.view(np.int32)).cuda()
                o2, _ = mq.attn_fwd(qd, kd, quant, md, w.causal)
                out[name] = _err(o2, ref, sel)
                out[name]["bf16_pairs"] = int(sum(bin(int(x)).count("1") for x in m.ravel()))
            out["bp500"]["bf16_pairs"] = int(cnt.sum())
    st, word = mq.device_status()
    assert st == 0, f"device watchdog raised {word:#x}"
    e0, e5, e100 = (out[f"bp{b}"]["rel_l2"] for b in (0, 500, 10000))
    out["gap_recovered"] = (e0 - e5) / (e0 - e100)
    out["gap_recovered_random"] = (e0 - out["bp500_random"]["rel_l2"]) / (e0 - e100)
    out["gap_recovered_forced_only"] = (e0 - out["forced_only"]["rel_l2"]) / (e0 - e100)
    out["gap_recovered_vertical_mode"] = (e0 - out["bp500_vertical_mode"]["rel_l2"]) / (e0 - e100)
    out["rows"] = int(sel.sum())
    assert e100 < e0
    return out


def test_quality_llm8k_full():
    _RESULTS["llm8k"] = _quality(workloads.WORKLOADS["llm8k"])


def test_quality_llm32k_sampled():
    w = workloads.WORKLOADS["llm32k"]
    _RESULTS["llm32k_64tiles"] = _quality(w, workloads.sample_query_tiles(w, 64, seed=1))


def test_quality_llm8k_planted_vertical_lines():
    """Structure away from the sink: the pooled score has to find the planted key tiles."""
    _RESULTS["llm8k_vlines"] = _quality(workloads.VLINES)


def test_quality_vit():
    _RESULTS["vit"] = _quality(workloads.WORKLOADS["vit"])


def teardown_module(module):
    path = os.environ.get("THRIFT_QUALITY_OUT")
    if path and _RESULTS:
        with open(path, "w") as f:
            json.dump(_RESULTS, f, indent=1)
