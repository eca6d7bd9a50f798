"""Pins for the oracle's NVFP4 (Q, K) and per-channel FP8 (V) quantisation.

Each pin is a property the NVFP4 recipe fixes independently of how the
oracle computes it: the per-element error bound of round-to-nearest on the
e2m1 grid, the block maximum landing on the top grid value, the head maximum
getting the largest block scale, exact power-of-two rescaling of V and the
minimality of its exponent.
"""
import numpy as np
import torch

from mixed_precision_bit_quant_b200 import workloads
from oracle.formats import e2m1_decode, e4m3_decode
from oracle.quantize import (fp8_v_quantize, nvfp4_dequantize, nvfp4_quantize,
                             pack_nibbles, unpack_nibbles, v_channel_exponent)


def _bf16(a):
    return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)


def _inputs():
    w = workloads.WORKLOADS["tiny"]
    q, k, v = workloads.generate(w)
    return q, k, v


def _half_spacing(y):
    a = np.abs(y)
    return np.where(a < 2.0, 0.25, np.where(a < 4.0, 0.5, 1.0))


def test_nvfp4_error_bound_per_element():
    q, k, _ = _inputs()
    for x in (q, k):
        codes, sf, g = nvfp4_quantize(x)
        xh = nvfp4_dequantize(codes, sf, g)
        xf = x.double().numpy()
        B, H, N, d = xf.shape
        den = (e4m3_decode(sf) * g[:, :, None, None].astype(np.float64))[..., None]
        den = np.broadcast_to(den, (B, H, N, d // 16, 16)).reshape(B, H, N, d)
        y = xf / den
        bound = _half_spacing(np.minimum(np.abs(y), 6.0)) * den * (1 + 1e-6)
        err = np.abs(xf - xh)
        sat = np.abs(y) > 6.0
        assert np.all(err[~sat] <= bound[~sat])
        # saturated elements are clipped to 6 * den and stay within one top-bin spacing
        assert np.all(err[sat] <= 1.0 * den[sat] * (1 + 1e-6))


def test_nvfp4_block_max_lands_on_six():
    q, k, _ = _inputs()
    for x in (q, k):
        codes, sf, g = nvfp4_quantize(x)
        xf = x.float().numpy()
        B, H, N, d = xf.shape
        blk = np.abs(xf.reshape(B, H, N, d // 16, 16))
        arg = blk.argmax(axis=4)
        c = np.take_along_axis(codes.reshape(B, H, N, d // 16, 16), arg[..., None], axis=4)[..., 0]
        normal = ((sf >> 3) & 0xF) >= 1
        nz = blk.max(axis=4) > 0
        sel = normal & nz
        assert sel.any()
        assert np.all((c[sel] & 7) == 7)               # magnitude 6 on the e2m1 grid


def test_nvfp4_head_max_gets_largest_scale():
    q, _, _ = _inputs()
    codes, sf, g = nvfp4_quantize(q)
    xf = np.abs(q.float().numpy())
    B, H, N, d = xf.shape
    amax = xf.reshape(B, H, -1).max(axis=2)
    assert np.allclose(g, amax / 2688.0, rtol=1e-7)
    for b in range(B):
        for h in range(H):
            n, c = np.unravel_index(np.argmax(xf[b, h]), (N, d))
            assert e4m3_decode(sf[b, h, n, c // 16]) == 448.0


def test_nvfp4_zero_head_and_zero_block():
    x = np.zeros((1, 2, 16, 32), dtype=np.float32)
    x[0, 1, 3, 17] = 1.5                                   # head 1 non-zero, block (3,1) only
    codes, sf, g = nvfp4_quantize(_bf16(x))
    assert g[0, 0] == 1.0 and np.all(codes[0, 0] == 0) and np.all(sf[0, 0] == 0)
    assert np.count_nonzero(sf[0, 1]) == 1 and e4m3_decode(sf[0, 1, 3, 1]) == 448.0
    assert e2m1_decode(codes[0, 1, 3, 17]) == 6.0
    # g = 1.5 / 2688 is rounded to FP32, so the dequantised value is 1.5 to FP32 precision
    assert abs(nvfp4_dequantize(codes, sf, g)[0, 1, 3, 17] - 1.5) <= 1.5 * 2.0 ** -23


def test_nvfp4_exact_on_representable_values():
    # a block whose values are e2m1 grid points times a power of two is reproduced exactly
    # head amax 6 * 448 * 2**-10 makes g = 2**-10 exact; that block gets scale 448, the others
    # (grid * 2**-3) get scale 2**-3 / g = 128: every value is code * scale * g exactly
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -6, -4, -3, -2, -1.5, -1, -0.5, 6], dtype=np.float32)
    x = np.tile(grid * 0.125, (1, 1, 4, 2))                # [1,1,4,32]
    x[0, 0, 0, :16] = grid * 448.0 * 2.0 ** -10
    codes, sf, g = nvfp4_quantize(_bf16(x))
    assert np.array_equal(nvfp4_dequantize(codes, sf, g), x.astype(np.float64))


def test_v_scale_exact_and_minimal():
    _, _, v = _inputs()
    v_code, v_exp, v_s = fp8_v_quantize(v)
    vf = v.double().numpy()
    e = v_exp.astype(np.int64)
    assert np.array_equal(np.ldexp(v_s.astype(np.float64), e[:, :, None, :]), vf)
    amax = np.abs(vf).max(axis=2)
    assert np.all(amax <= 448.0 * np.ldexp(1.0, e))
    assert np.all(amax > 448.0 * np.ldexp(1.0, e - 1))
    assert np.all(np.abs(e4m3_decode(v_code)) <= 448.0)
    # v_s is BF16-exact
    assert np.array_equal(torch.tensor(v_s).to(torch.bfloat16).float().numpy(), v_s)


def test_v_channel_exponent_edges():
    a = np.array([0.0, 448.0, 448.0001, 224.0, 1.0, 896.0, 897.0, 2.0 ** -20])
    e = v_channel_exponent(a)
    assert list(e[:7]) == [0, 0, 1, -1, -8, 1, 2]
    for x, ee in zip(a[1:], e[1:]):
        assert x <= 448 * 2.0 ** ee and x > 448 * 2.0 ** (ee - 1)


def test_nibble_packing_roundtrip(rng):
    c = rng.integers(0, 16, size=(3, 64)).astype(np.uint8)
    p = pack_nibbles(c)
    assert p[0, 0] == (c[0, 0] | (c[0, 1] << 4))
    assert np.array_equal(unpack_nibbles(p), c)


def test_v_copy_rounds_bf16_subnormals_to_nearest_even():
    """A channel whose maximum is far above its other values: v * 2**-e_c falls into the
    BF16 subnormals (spacing 2**-133), where the copy rounds to the nearest grid point
    with ties to even and keeps the sign; the e4m3 codes of those values are +-0."""
    amax = 2.0 ** 127                     # e_c = 119: 2**127 <= 448 * 2**119
    tiny = np.array([0.25, 0.375, 0.5, 0.75, 1.0, 1.25, 1.5, 2.5, 3.0, 100.0], dtype=np.float64)
    vals = np.concatenate([[amax], tiny * 2.0 ** -14, -tiny * 2.0 ** -14])  # all BF16 values
    v = torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).reshape(1, 1, -1, 1)
    assert np.array_equal(v.double().numpy().ravel(), vals)
    v_code, v_exp, v_s = fp8_v_quantize(v)
    assert int(v_exp[0, 0, 0]) == 119
    exact = vals * 2.0 ** -119            # the tiny ones: 0.25 .. 100 times 2**-133
    step = 2.0 ** -133
    # brute-force nearest grid point, ties to the even multiple
    k = np.floor(np.abs(exact) / step)
    frac = np.abs(exact) / step - k
    up = (frac > 0.5) | ((frac == 0.5) & (k % 2 == 1))
    want = np.sign(exact) * (k + up) * step
    got = v_s.astype(np.float64).ravel()
    assert np.array_equal(got[1:], want[1:])
    assert np.array_equal(np.signbit(got[1:]), np.signbit(exact[1:]))   # -0 kept
    assert got[0] == 256.0
    # the e4m3 codes of the tiny values are zeros with their signs
    codes = v_code.ravel()[1:]
    assert np.array_equal(codes, np.where(exact[1:] < 0, 0x80, 0x00))
