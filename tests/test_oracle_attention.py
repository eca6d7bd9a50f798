"""Pins for the oracle's mixed-precision tiled attention.

The method reduces to textbook softmax attention in its special cases:
* all tiles BF16 and no P rounding: exact softmax attention on the inputs;
* no tile BF16 and no P rounding: exact softmax attention on the
  dequantised NVFP4 Q, K and FP8 V;
* any mask, no P rounding: one softmax over the logit matrix assembled
  tile by tile from the two precisions (the "single output" of the online
  merge);
* V = 1: the effective probabilities of every row sum to one;
* Q = 0: uniform weights, the output is the (prefix) mean of V';
* one key: the output is that key's value row.
"""
import math

import numpy as np
import pytest
import torch

from oracle.attention import attn_forward, exact_attention
from oracle.formats import e4m3_decode
from oracle.quantize import nvfp4_dequantize, quantize
from oracle.select import mask_to_dense, select


def _problem(B=1, Hq=4, Hkv=2, N=300, d=64, seed=0, scale_q=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (scale_q * torch.randn((B, Hq, N, d), generator=g)).to(torch.bfloat16)
    k = (torch.randn((B, Hkv, N, d), generator=g) + 0.3).to(torch.bfloat16)
    v = torch.randn((B, Hkv, N, d), generator=g).to(torch.bfloat16)
    return q, k, v


def _full_mask(B, H, T, value):
    W = (T + 31) // 32
    m = np.zeros((B, H, T, W), dtype=np.uint32)
    if value:
        for j in range(T):
            m[..., j // 32] |= np.uint32(1) << np.uint32(j % 32)
    return m


@pytest.mark.parametrize("causal", [False, True])
def test_all_bf16_equals_exact_attention(causal):
    q, k, v = _problem()
    qz = quantize(q, k, v)
    T = 3
    O, _ = attn_forward(q, k, v, qz, _full_mask(1, 4, T, True), causal, p_cast=False)
    ref = exact_attention(q, k, v, causal)
    assert np.max(np.abs(O - ref)) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_all_fp4_equals_attention_on_dequantised_inputs(causal):
    q, k, v = _problem(seed=1)
    qz = quantize(q, k, v)
    T = 3
    O, _ = attn_forward(q, k, v, qz, _full_mask(1, 4, T, False), causal, p_cast=False)
    qh = nvfp4_dequantize(qz["q_codes"], qz["q_sf"], qz["q_g"])
    kh = nvfp4_dequantize(qz["k_codes"], qz["k_sf"], qz["k_g"])
    vh = e4m3_decode(qz["v_code"]) * np.ldexp(1.0, qz["v_exp"].astype(np.int64))[:, :, None, :]
    ref = exact_attention(qh, kh, vh, causal)
    assert np.max(np.abs(O - ref)) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_online_merge_equals_one_softmax_over_mixed_logits(causal):
    B, Hq, Hkv, N, d = 1, 4, 2, 300, 64
    q, k, v = _problem(B, Hq, Hkv, N, d, seed=2)
    qz = quantize(q, k, v)
    sel = select(q, k, causal, budget_bp=3000)
    T = 3
    O, lse = attn_forward(q, k, v, qz, sel["mask"], causal, p_cast=False)
    dense = mask_to_dense(sel["mask"], T)
    qh = nvfp4_dequantize(qz["q_codes"], qz["q_sf"], qz["q_g"])
    kh = nvfp4_dequantize(qz["k_codes"], qz["k_sf"], qz["k_g"])
    vh = e4m3_decode(qz["v_code"]) * np.ldexp(1.0, qz["v_exp"].astype(np.int64))[:, :, None, :]
    qf, kf, vf = (t.double().numpy() for t in (q, k, v))
    G = Hq // Hkv
    for h in range(Hq):
        hk = h // G
        S_hi = qf[0, h] @ kf[0, hk].T / math.sqrt(d)
        S_lo = qh[0, h] @ kh[0, hk].T / math.sqrt(d)
        tile_hi = np.kron(dense[0, h].astype(int), np.ones((128, 128), dtype=int))[:N, :N].astype(bool)
        S = np.where(tile_hi, S_hi, S_lo)
        if causal:
            S = np.where(np.tril(np.ones((N, N), dtype=bool)), S, -np.inf)
        P = np.exp(S - S.max(axis=1, keepdims=True))
        P = P / P.sum(axis=1, keepdims=True)
        # each key's value row comes from the precision of its tile pair
        ref = (P * tile_hi) @ vf[0, hk] + (P * ~tile_hi) @ vh[0, hk]
        assert np.max(np.abs(O[0, h] - ref)) < 1e-12
        lse_ref = np.log(np.sum(np.exp(S - S.max(axis=1, keepdims=True)), axis=1)) + S.max(axis=1)
        assert np.max(np.abs(lse[0, h] - lse_ref)) < 1e-10


@pytest.mark.parametrize("p_cast", [False, True])
def test_probability_rows_sum_to_one(p_cast):
    q, k, _ = _problem(seed=3)
    v = torch.ones((1, 2, 300, 64), dtype=torch.bfloat16)
    qz = quantize(q, k, v)
    assert np.all(e4m3_decode(qz["v_code"]) * np.ldexp(1.0, qz["v_exp"].astype(np.int64))[:, :, None, :] == 1.0)
    sel = select(q, k, True, budget_bp=2000)
    O, _ = attn_forward(q, k, v, qz, sel["mask"], True, p_cast=p_cast)
    if p_cast:
        # every cast p is within half an e4m3 step (2**-4 relative) or the subnormal step
        assert np.max(np.abs(O - 1.0)) <= 2.0 ** -4
    else:
        assert np.max(np.abs(O - 1.0)) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_mean_of_values(causal):
    q, k, v = _problem(seed=4, scale_q=0.0)
    qz = quantize(q, k, v)
    sel = select(q, k, causal, budget_bp=5000)
    O, _ = attn_forward(q, k, v, qz, sel["mask"], causal, p_cast=True)
    dense = mask_to_dense(sel["mask"], 3)
    vf = v.double().numpy()
    vh = e4m3_decode(qz["v_code"]) * np.ldexp(1.0, qz["v_exp"].astype(np.int64))[:, :, None, :]
    N = 300
    for h in range(4):
        hk = h // 2
        for r in (0, 5, 127, 128, 200, 299):
            n_keys = r + 1 if causal else N
            rows = [vf[0, hk, j] if dense[0, h, r // 128, j // 128] else vh[0, hk, j] for j in range(n_keys)]
            assert np.allclose(O[0, h, r], np.mean(rows, axis=0), rtol=0, atol=1e-12)


def test_single_key():
    q, k, v = _problem(N=1, seed=5)
    qz = quantize(q, k, v)
    for hi in (False, True):
        O, lse = attn_forward(q, k, v, qz, _full_mask(1, 4, 1, hi), True, p_cast=True)
        for h in range(4):
            want = v.double().numpy()[0, h // 2, 0] if hi else \
                e4m3_decode(qz["v_code"][0, h // 2, 0]) * np.ldexp(1.0, qz["v_exp"][0, h // 2].astype(np.int64))
            assert np.allclose(O[0, h, 0], want, atol=1e-12)


def test_sampled_tiles_match_full_run():
    q, k, v = _problem(N=400, seed=6)
    qz = quantize(q, k, v)
    sel = select(q, k, True, budget_bp=500)
    O, _ = attn_forward(q, k, v, qz, sel["mask"], True)
    Os, _ = attn_forward(q, k, v, qz, sel["mask"], True, tiles=[(0, 1, 2), (0, 3, 0)])
    assert np.array_equal(Os[0, 1, 256:384], O[0, 1, 256:384])
    assert np.array_equal(Os[0, 3, 0:128], O[0, 3, 0:128])
    assert np.isnan(Os[0, 0]).all()


def test_on_demand_quantisation_matches_full_quantisation():
    q, k, v = _problem(N=400, seed=8)
    qz = quantize(q, k, v)
    sel = select(q, k, True, budget_bp=1500)
    tiles = [(0, 0, 3), (0, 2, 1), (0, 3, 2)]
    O1, l1 = attn_forward(q, k, v, qz, sel["mask"], True, tiles=tiles)
    O2, l2 = attn_forward(q, k, v, None, sel["mask"], True, tiles=tiles)
    assert np.array_equal(np.nan_to_num(O1, nan=7.0), np.nan_to_num(O2, nan=7.0))


@pytest.mark.parametrize("causal", [False, True])
def test_exact_attention_tiles_is_exact_attention_row_by_row(causal):
    from oracle.attention import exact_attention_tiles
    q, k, v = _problem(N=300, seed=9)
    ref = exact_attention(q, k, v, causal)
    tiles = [(0, 0, 0), (0, 1, 2), (0, 3, 1)]
    O = exact_attention_tiles(q, k, v, causal, tiles)
    for (b, h, i) in tiles:
        r0, r1 = i * 128, min(300, (i + 1) * 128)
        assert np.max(np.abs(O[b, h, r0:r1] - ref[b, h, r0:r1])) < 1e-12
    assert np.isnan(O[0, 2]).all()
    # first row of a causal problem sees one key: its value row
    if causal:
        assert np.allclose(O[0, 0, 0], v.double().numpy()[0, 0, 0], atol=0)
