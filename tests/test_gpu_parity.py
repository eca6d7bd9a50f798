"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bar: bit-exact codes, scales, exponents and masks; attention outputs within
max|err| <= 2e-2 * max|O_ref| and relative L2 <= 5e-3 of the oracle on the
same seeded inputs.  Inputs are drawn on the host and copied to the device,
so both sides see identical bytes; no expected value comes from the GPU.
"""
import numpy as np
import pytest
import torch

import mixed_precision_bit_quant_b200 as mq
from mixed_precision_bit_quant_b200 import workloads
from oracle import attention as oatt
from oracle import quantize as oq
from oracle import select as osel

pytestmark = pytest.mark.gpu

MAX_ERR = 2e-2
REL_L2 = 5e-3


def _cuda(*ts):
    return tuple(t.cuda() for t in ts)


def _unswizzle_sf(mma: np.ndarray, B, H, T, d) -> np.ndarray:
    """[B,H,T,d/64,512] tensor-core scale layout -> [B,H,T*128,d/16] row-major."""
    KB = d // 64
    a = mma.reshape(B, H, T, KB, 32, 4, 4)            # (t, kb, r0, r1, k)
    a = a.transpose(0, 1, 2, 5, 4, 3, 6)              # (t, r1, r0, kb, k)
    return a.reshape(B, H, T * 128, KB * 4)


def check_quantize(q, k, v, got: dict):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    T = (N + 127) // 128
    Np = T * 128
    ref = oq.quantize(q, k, v)
    g = {f: t.cpu() for f, t in got.items()}
    for side, H in (("q", Hq), ("k", Hkv)):
        codes = g[f"{side}_fp4"].numpy().reshape(B, H, N, d // 2)
        assert np.array_equal(codes, oq.pack_nibbles(ref[f"{side}_codes"])), f"{side} codes"
        sf = g[f"{side}_sf"].numpy().reshape(B, H, N, d // 16)
        assert np.array_equal(sf, ref[f"{side}_sf"]), f"{side} scales"
        mma = _unswizzle_sf(g[f"{side}_sf_mma"].numpy(), B, H, T, d)
        assert np.array_equal(mma[:, :, :N], ref[f"{side}_sf"]), f"{side} tensor-core scales"
        assert not mma[:, :, N:].any()
        gs = g[f"{side}_gs"].numpy().reshape(B, H)
        assert np.array_equal(gs.view(np.uint32), ref[f"{side}_g"].view(np.uint32)), f"{side} tensor scale"
    vt = g["v_fp8t"].numpy().reshape(B, Hkv, d, Np)
    assert np.array_equal(vt[..., :N].transpose(0, 1, 3, 2), ref["v_code"]), "v codes"
    assert not vt[..., N:].any()
    vs = g["v_st"].float().numpy().reshape(B, Hkv, d, Np)
    assert np.array_equal(vs[..., :N].transpose(0, 1, 3, 2), ref["v_s"]), "v bf16 copy"
    assert np.array_equal(g["v_exp"].numpy().reshape(B, Hkv, d), ref["v_exp"]), "v exponents"


def check_close(o_gpu: np.ndarray, o_ref: np.ndarray, what: str):
    assert np.isfinite(o_gpu).all(), what
    err = np.abs(o_gpu - o_ref)
    mx = np.abs(o_ref).max()
    rel = np.linalg.norm(o_gpu - o_ref) / np.linalg.norm(o_ref)
    assert err.max() <= MAX_ERR * mx, f"{what}: max err {err.max():.3e} vs {MAX_ERR * mx:.3e}"
    assert rel <= REL_L2, f"{what}: rel L2 {rel:.3e}"
    return float(err.max() / mx), float(rel)


def run_case(q, k, v, causal, bp, tiles_budget, sample=None, check_quant=True):
    """Run the three calls on the GPU and compare each stage with the oracle."""
    B, Hq, N, d = q.shape
    T = (N + 127) // 128
    qd, kd, vd = _cuda(q, k, v)
    quant = mq.quantize(qd, kd, vd)
    mask, counts = mq.select(qd, kd, causal, bp, tiles_budget)
    o, lse = mq.attn_fwd(qd, kd, quant, mask, causal, want_lse=True)
    st, word = mq.device_status()
    assert st == 0, f"device watchdog raised {word:#x}"
    if check_quant:
        check_quantize(q, k, v, quant.tensors)
    rows = sample
    ref_sel = osel.select(q, k, causal, bp, tiles_budget, rows=rows)
    gmask = mask.cpu().numpy().view(np.uint32)
    gcnt = counts.cpu().numpy()
    if rows is None:
        assert np.array_equal(gmask, ref_sel["mask"]), "mask"
        assert np.array_equal(gcnt, ref_sel["counts"]), "counts"
    else:
        for (b, h, i) in rows:
            assert np.array_equal(gmask[b, h, i], ref_sel["mask"][b, h, i]), ("mask", b, h, i)
            assert gcnt[b, h, i] == ref_sel["counts"][b, h, i]
    O_ref, lse_ref = oatt.attn_forward(q, k, v, None, ref_sel["mask"], causal, tiles=rows)
    og = o.float().cpu().numpy().astype(np.float64)
    lg = lse.cpu().numpy().astype(np.float64)
    if rows is None:
        res = check_close(og, O_ref, "O")
        assert np.max(np.abs(lg - lse_ref)) < 1e-3
    else:
        sel = np.zeros(O_ref.shape[:3], dtype=bool)
        for (b, h, i) in rows:
            sel[b, h, i * 128:min(N, (i + 1) * 128)] = True
        res = check_close(og[sel], O_ref[sel], "O (sampled tiles)")
        assert np.max(np.abs(lg[sel] - lse_ref[sel])) < 1e-3
    return res


def test_tiny_workload():
    w = workloads.WORKLOADS["tiny"]
    q, k, v = workloads.generate(w)
    run_case(q, k, v, w.causal, w.budget_bp, w.budget_tiles)


def test_vit_workload_ragged():
    w = workloads.WORKLOADS["vit"]
    q, k, v = workloads.generate(w)
    run_case(q, k, v, w.causal, w.budget_bp, w.budget_tiles)


def test_llm8k_workload_full():
    w = workloads.WORKLOADS["llm8k"]
    q, k, v = workloads.generate(w)
    run_case(q, k, v, w.causal, w.budget_bp, w.budget_tiles, check_quant=True)


@pytest.mark.parametrize("bp", [0, 500, 10000])
def test_llm32k_sampled_tiles(bp):
    w = workloads.WORKLOADS["llm32k"].with_budget(bp=bp)
    q, k, v = workloads.generate(w)
    sample = workloads.sample_query_tiles(w, 64, seed=1)
    run_case(q, k, v, w.causal, w.budget_bp, w.budget_tiles, sample=sample, check_quant=(bp == 500))


def test_llm128k_sampled_tiles():
    w = workloads.WORKLOADS["llm128k"]
    q, k, v = workloads.generate(w)
    sample = workloads.sample_query_tiles(w, 64, seed=1)
    run_case(q, k, v, w.causal, w.budget_bp, w.budget_tiles, sample=sample, check_quant=False)


@pytest.mark.parametrize("N,d,Hq,Hkv,causal,bp,bt", [
    (1, 128, 4, 2, True, 500, 0),        # one key
    (1, 64, 2, 2, False, 0, 0),
    (129, 128, 4, 1, True, 3000, 0),     # one-row ragged tail, GQA 4
    (200, 64, 6, 3, False, 10000, 0),    # all BF16
    (640, 128, 8, 2, True, 0, 0),        # all FP4
    (640, 128, 8, 2, False, 0, 3),
    (1000, 64, 4, 4, True, 2500, 0),
    (1536, 128, 2, 1, False, 700, 0),
])
def test_shapes_and_budgets(N, d, Hq, Hkv, causal, bp, bt):
    w = workloads.custom("case", 1, Hq, Hkv, N, d, causal, "llm", bp, bt, seed=N + d)
    q, k, v = workloads.generate(w)
    run_case(q, k, v, causal, bp, bt)


def test_zero_head_and_batch():
    w = workloads.custom("zero", 2, 4, 2, 300, 128, True, "llm", 2000, 0, seed=3)
    q, k, v = workloads.generate(w)
    q[0, 1] = 0
    k[1, 0] = 0
    run_case(q, k, v, True, 2000, 0)


def test_lse_optional_and_repeatable():
    w = workloads.custom("rep", 1, 4, 2, 700, 128, True, "llm", 500, 0, seed=5)
    q, k, v = _cuda(*workloads.generate(w))
    o1, _ = mq.attention(q, k, v, True, 500)
    o2, lse = mq.attention(q, k, v, True, 500, want_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)                 # deterministic
    assert lse is not None and torch.isfinite(lse).all()


def test_p_cast_closed_forms_on_gpu():
    """The hand-derived P-cast cases of tests/golden/p_cast_closed_forms.txt through the C ABI."""
    from tests.test_golden import p_cast_cases, p_cast_problem
    for name, tile, e_t, o0, o1 in p_cast_cases():
        q, k, v, scale = p_cast_problem(e_t)
        qd, kd, vd = _cuda(q, k, v)
        quant = mq.quantize(qd, kd, vd)
        mask = torch.full((1, 1, 1, 1), 1 if tile == "bf16" else 0, dtype=torch.int32, device="cuda")
        o, _ = mq.attn_fwd(qd, kd, quant, mask, False, softmax_scale=scale)
        st, word = mq.device_status()
        assert st == 0, f"device watchdog raised {word:#x}"
        og = o.float().cpu().numpy()[0, 0]
        # only the BF16 rounding of the output separates the kernel from the closed form
        for got, want in ((og[0, 0], float(o0)), (og[0, 1], float(o1))):
            assert abs(got - want) <= 2.0 ** -8 * want, (name, got, want)
        assert not og[0, 2:].any()
        assert np.allclose(og[1, :2], 0.5, rtol=0, atol=0) and not og[1, 2:].any()


@pytest.mark.parametrize("scale", [0.05, 0.2])
def test_custom_softmax_scale(scale):
    """A softmax scale other than 1/sqrt(d) on both tile kinds (the FP4 path folds the
    tensor scales of Q and K into it)."""
    w = workloads.custom("scale", 1, 4, 2, 700, 128, True, "llm", 3000, 0, seed=11)
    q, k, v = workloads.generate(w)
    qd, kd, vd = _cuda(q, k, v)
    quant = mq.quantize(qd, kd, vd)
    mask, _ = mq.select(qd, kd, True, 3000)
    o, lse = mq.attn_fwd(qd, kd, quant, mask, True, softmax_scale=scale, want_lse=True)
    st, word = mq.device_status()
    assert st == 0, f"device watchdog raised {word:#x}"
    ref_sel = osel.select(q, k, True, 3000)
    assert np.array_equal(mask.cpu().numpy().view(np.uint32), ref_sel["mask"])
    O_ref, lse_ref = oatt.attn_forward(q, k, v, None, ref_sel["mask"], True, sm_scale=scale)
    check_close(o.float().cpu().numpy().astype(np.float64), O_ref, f"O (scale {scale})")
    assert np.max(np.abs(lse.cpu().numpy() - lse_ref)) < 1e-3
