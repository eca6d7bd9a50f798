"""GPU parity of the microscaling variant: MXFP4 Q and K (thrift_quantize_mx,
thrift_attn_fwd_mx) against the oracle (oracle/mx.py; the attention-
quantization topic page lists MXFP4 beside NVFP4 and a diagonal-tiled
mixed-precision MXFP method).

Bar: e2m1 codes, e8m0 scales (row-major and tensor-core order) and the V
operands bit-exact; the output within max|err| <= 2e-2 * max|O_ref| and
relative L2 <= 5e-3 of ``oracle.attention.attn_forward(fmt="mxfp4_qk")`` on
the same seeded inputs, with the mask from thrift_select.
"""
import numpy as np
import pytest
import torch

import mixed_precision_bit_quant_b200 as mq
from mixed_precision_bit_quant_b200 import workloads
from oracle import attention as oatt
from oracle import mx
from oracle import quantize as oq
from oracle import select as osel

pytestmark = pytest.mark.gpu


def _mma_chunks(sc: np.ndarray, T: int) -> np.ndarray:
    """[B,H,N,d/32] e8m0 codes -> [B,H,T,d/64,512]: per K=64 step, word 16*(r%32)+4*(r/32)
    holds row r's two block scales in bytes 0 and 1."""
    B, H, N, nb = sc.shape
    ref = np.zeros((B, H, T, nb // 2, 512), np.uint8)
    r = np.arange(N)
    t, rr = r // 128, r % 128
    off = (rr % 32) * 16 + (rr // 32) * 4
    for kb in range(nb // 2):
        view = ref[:, :, :, kb, :]                  # [B, H, T, 512]
        for byte in range(2):
            view[:, :, t, off + byte] = sc[:, :, :, 2 * kb + byte]
    return ref


def _check_quant(q, k, v, quant):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    T = (N + 127) // 128
    g = {f: t.cpu().numpy() for f, t in quant.tensors.items() if t.dtype != torch.bfloat16}
    for side, x, H in (("q", q, Hq), ("k", k, Hkv)):
        codes, sc = mx.mx_quantize(x, "e2m1", axis=3)
        assert np.array_equal(g[f"{side}_fp4"].reshape(B, H, N, d // 2), oq.pack_nibbles(codes)), f"{side} codes"
        assert np.array_equal(g[f"{side}_sf"][: sc.size].reshape(sc.shape), sc), f"{side} e8m0 scales"
        got = g[f"{side}_sf_mma"].reshape(B, H, T, d // 64, 512)
        assert np.array_equal(got, _mma_chunks(sc, T)), f"{side} tensor-core scales"
        assert np.all(g[f"{side}_gs"] == 1.0)
    ref = oq.quantize(q, k, v)
    Np = T * 128
    vt = g["v_fp8t"].reshape(B, Hkv, d, Np)
    assert np.array_equal(vt[..., :N].transpose(0, 1, 3, 2), ref["v_code"]), "v codes"
    assert np.array_equal(g["v_exp"].reshape(B, Hkv, d), ref["v_exp"]), "v exponents"


def _run(w, sample=None, check_quant=True):
    q, k, v = workloads.generate(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    quant = mq.quantize(qd, kd, vd, fmt="mxfp4")
    mask, _ = mq.select(qd, kd, w.causal, w.budget_bp, w.budget_tiles)
    o, lse = mq.attn_fwd(qd, kd, quant, mask, w.causal, want_lse=True)
    st, word = mq.device_status()
    assert st == 0, f"device watchdog raised {word:#x}"
    if check_quant:
        _check_quant(q, k, v, quant)
    m = mask.cpu().numpy().view(np.uint32)
    ref_sel = osel.select(q, k, w.causal, w.budget_bp, w.budget_tiles, rows=sample)
    if sample is None:
        assert np.array_equal(m, ref_sel["mask"])
    O_ref, lse_ref = oatt.attn_forward(q, k, v, None, m, w.causal, tiles=sample, fmt="mxfp4_qk")
    sel = ~np.isnan(O_ref[..., 0])
    og = o.float().cpu().numpy().astype(np.float64)[sel]
    r = O_ref[sel]
    err = np.abs(og - r).max() / np.abs(r).max()
    rel = np.linalg.norm(og - r) / np.linalg.norm(r)
    assert err <= 2e-2 and rel <= 5e-3, (err, rel)
    assert np.max(np.abs(lse.cpu().numpy()[sel] - lse_ref[sel])) < 1e-3


@pytest.mark.parametrize("name", ["tiny", "vit", "llm8k"])
def test_mx_workloads(name):
    _run(workloads.WORKLOADS[name])


def test_mx_llm32k_sampled_all_fp4():
    w = workloads.WORKLOADS["llm32k"].with_budget(bp=0)
    _run(w, sample=workloads.sample_query_tiles(w, 32, seed=1), check_quant=False)


@pytest.mark.parametrize("N,d,Hq,Hkv,causal,bp", [
    (1, 128, 2, 1, True, 0),
    (129, 64, 4, 2, True, 0),
    (300, 64, 4, 2, True, 2500),
    (200, 128, 4, 2, False, 0),
    (640, 128, 8, 2, True, 500),
])
def test_mx_shapes(N, d, Hq, Hkv, causal, bp):
    _run(workloads.custom("mx", 1, Hq, Hkv, N, d, causal, "llm", bp, 0, seed=9 + N))


def test_mx_zero_blocks():
    w = workloads.custom("mxz", 1, 2, 1, 256, 128, True, "llm", 0, 0, seed=4)
    q, k, v = workloads.generate(w)
    q[0, 0, 5:9] = 0          # all-zero blocks take scale code 0 and zero codes
    k[0, 0, 100, :32] = 0
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    quant = mq.quantize(qd, kd, vd, fmt="mxfp4")
    mq.device_status()
    _check_quant(q, k, v, quant)
