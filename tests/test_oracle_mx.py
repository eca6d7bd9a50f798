"""Pins of the microscaling (MX) oracle, oracle/mx.py.

Each test checks the oracle against what the OCP microscaling definition and
plain arithmetic fix, not against a retyping of its own formulas: exact
decoding of every scale code, the shared exponent on values built with a
known binade, exact round trips of values the format can hold, brute-force
nearest grid points, the saturation the definition implies, and the
attention identity at a zero BF16 budget.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import mx
from oracle import select as osel

E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def test_e8m0_decode_every_code():
    for c in range(255):
        assert mx.e8m0_decode(c) == math.ldexp(1.0, c - 127)
    assert np.isnan(mx.e8m0_decode(255))


@pytest.mark.parametrize("emax", [2, 8])
def test_shared_exponent_on_known_binades(emax):
    rng = np.random.default_rng(1)
    for k in list(range(-140, 130, 7)) + [-149, -127, -126, 0, 127]:
        for m in (1.0, 1.0 + 2.0 ** -23, 1.5, 2.0 - 2.0 ** -23, float(rng.uniform(1, 2))):
            a = np.float32(math.ldexp(m, k))
            if a == 0 or not np.isfinite(a):
                continue
            kk = math.frexp(float(a))[1] - 1                  # binade of the float32 value
            want = min(127, max(-127, kk - emax))
            assert int(mx.mx_shared_exponent(a, emax)) == want, (a, emax)
    assert int(mx.mx_shared_exponent(0.0, emax)) == -127


def test_zero_block_gets_smallest_scale_and_zero_codes():
    x = np.zeros((1, 1, 3, 64), np.float32)
    x[0, 0, 1, 40] = -0.0
    codes, sc = mx.mx_quantize(x, "e2m1", axis=3)
    assert np.all(sc == 0)
    assert np.all((codes & 7) == 0)
    assert codes[0, 0, 1, 40] == 8          # sign of zero kept


def test_mxfp4_roundtrip_of_representable_blocks():
    # a block whose largest magnitude is 4 or 6 times 2**e has shared exponent e,
    # so every element of the form grid_value * 2**e is reproduced exactly
    rng = np.random.default_rng(2)
    for _ in range(200):
        e = int(rng.integers(-20, 20))
        idx = rng.integers(0, 8, size=32)
        idx[rng.integers(0, 32)] = rng.choice([6, 7])        # block max 4 or 6
        sign = rng.integers(0, 2, size=32)
        vals = np.where(sign == 1, -1.0, 1.0) * E2M1_VALUES[idx] * 2.0 ** e
        codes, sc = mx.mx_quantize(vals.reshape(1, 1, 1, 32).astype(np.float32), "e2m1", axis=3)
        assert int(sc.ravel()[0]) == e + 127
        back = mx.mx_dequantize(codes, sc, "e2m1", axis=3).ravel()
        assert np.array_equal(back, vals)


def test_mxfp4_is_nearest_grid_point_or_saturated():
    # brute force over the grid: every element lands on a nearest grid point of
    # the block's scale (ties to the even code), or on +-6 X when |x| / X > 6
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((4, 3, 50, 64)) * np.exp(rng.uniform(-6, 6, (4, 3, 50, 1)))).astype(np.float32)
    codes, sc = mx.mx_quantize(x, "e2m1", axis=3)
    xh = mx.mx_dequantize(codes, sc, "e2m1", axis=3)
    X = np.repeat(mx.e8m0_decode(sc), 32, axis=3)
    y = np.abs(x.astype(np.float64)) / X
    assert np.all(y < 8)                                      # amax / X in [4, 8)
    grid = E2M1_VALUES[None, :]
    flat_y, flat_h = y.ravel(), np.abs(xh).ravel() / X.ravel()
    dist = np.abs(flat_y[:, None] - grid)
    best = dist.min(axis=1)
    inside = flat_y <= 6
    assert np.all(np.abs(np.abs(flat_h[inside] - flat_y[inside]) - best[inside]) == 0)
    assert np.all(flat_h[~inside] == 6)
    assert np.array_equal(np.signbit(xh), np.signbit(x))


def test_mxfp8_roundtrip_and_saturation():
    rng = np.random.default_rng(4)
    # representable: e4m3 normal values times 2**e with a block max in [256, 448]
    for _ in range(100):
        e = int(rng.integers(-30, 10))
        m = rng.integers(8, 16, size=32)                      # 1.m mantissa * 8
        ex = rng.integers(-6, 9, size=32)
        ex[0] = 8                                             # block max in [256, 448]
        m = np.where(ex == 8, np.minimum(m, 14), m)           # 1.875 * 2**8 = 480 is not an e4m3 value
        vals = (m / 8.0) * np.ldexp(1.0, ex) * 2.0 ** e
        v = vals.reshape(1, 1, 32, 1).astype(np.float32)
        codes, sc = mx.mx_quantize(v, "e4m3", axis=2)
        assert int(sc.ravel()[0]) == e + 127
        assert np.array_equal(mx.mx_dequantize(codes, sc, "e4m3", axis=2).ravel(), vals)
    # a block maximum of 1.9 * 2**k is above 448 X and saturates to 448 X
    v = np.zeros((1, 1, 32, 1), np.float32)
    v[0, 0, 5, 0] = 1.9 * 2.0 ** 3
    codes, sc = mx.mx_quantize(v, "e4m3", axis=2)
    assert int(sc.ravel()[0]) == 3 - 8 + 127
    assert mx.mx_dequantize(codes, sc, "e4m3", axis=2)[0, 0, 5, 0] == 448.0 * 2.0 ** -5


def test_ragged_key_blocks_use_valid_keys_only():
    rng = np.random.default_rng(5)
    v = rng.standard_normal((1, 2, 70, 8)).astype(np.float32)
    codes, sc = mx.mx_quantize(v, "e4m3", axis=2)
    assert sc.shape == (1, 2, 3, 8)
    last = np.abs(v[:, :, 64:70, :].astype(np.float64)).max(axis=2)
    assert np.array_equal(sc[:, :, 2, :].astype(np.int64), mx.mx_shared_exponent(last, 8) + 127)
    # quantising the valid part alone gives the same codes
    c2, s2 = mx.mx_quantize(v[:, :, 64:70, :], "e4m3", axis=2)
    assert np.array_equal(c2, codes[:, :, 64:70, :]) and np.array_equal(s2[:, :, 0], sc[:, :, 2])


@pytest.mark.parametrize("causal", [False, True])
def test_zero_budget_mx_attention_is_attention_on_dequantised_inputs(causal):
    g = torch.Generator().manual_seed(6)
    B, Hq, Hkv, N, d = 1, 4, 2, 300, 64
    q = torch.randn(B, Hq, N, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, N, d, generator=g).to(torch.bfloat16)
    quant = mx.quantize(q, k, v)
    qh, kh, vh = mx.dequantized(quant)
    mask = osel.select(q, k, causal, 0)["mask"]
    assert not mask.any()
    O, _ = oatt.attn_forward(q, k, v, quant, mask, causal, p_cast=False, fmt="mx")
    ref = oatt.exact_attention(qh, kh, vh, causal)
    assert np.abs(O - ref).max() < 1e-12


def test_mxfp4_midpoints_round_to_the_even_code():
    # block maximum 4 X fixes X; each midpoint between neighbouring grid values goes
    # to the neighbour with the even code (mantissa bit 0)
    e = -3
    X = 2.0 ** e
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    want = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    vals = np.zeros(32)
    vals[0] = 4.0 * X
    vals[1:1 + len(mids)] = np.array(mids) * X
    vals[10:10 + len(mids)] = -np.array(mids) * X
    codes, sc = mx.mx_quantize(vals.reshape(1, 1, 1, 32).astype(np.float32), "e2m1", axis=3)
    assert int(sc.ravel()[0]) == e + 127 and mx.e8m0_decode(sc.ravel()[0]) == X
    back = mx.mx_dequantize(codes, sc, "e2m1", axis=3).ravel() / X
    assert list(back[1:1 + len(mids)]) == want
    assert list(-back[10:10 + len(mids)]) == want


@pytest.mark.parametrize("causal", [False, True])
def test_zero_budget_mxfp4_qk_attention_keeps_channel_fp8_values(causal):
    # MXFP4 Q and K with V in the per-channel FP8 of the NVFP4 path: at a zero budget
    # without P rounding, softmax attention on (MX Q, MX K, channel-FP8 V)
    from oracle import formats, quantize as oq
    g = torch.Generator().manual_seed(7)
    B, Hq, Hkv, N, d = 1, 2, 1, 260, 64
    q = torch.randn(B, Hq, N, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, N, d, generator=g).to(torch.bfloat16)
    v = (torch.randn(B, Hkv, N, d, generator=g) * 3).to(torch.bfloat16)
    qh, kh, _ = mx.dequantized(mx.quantize(q, k, v))
    v_code, v_exp, _ = oq.fp8_v_quantize(v)
    vh = formats.e4m3_decode(v_code) * np.ldexp(1.0, v_exp.astype(np.int64))[:, :, None, :]
    mask = osel.select(q, k, causal, 0)["mask"]
    O, _ = oatt.attn_forward(q, k, v, None, mask, causal, p_cast=False, fmt="mxfp4_qk")
    assert np.abs(O - oatt.exact_attention(qh, kh, vh, causal)).max() < 1e-12
