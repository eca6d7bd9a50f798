"""Oracle: block-scaled quantisation of Q, K (NVFP4) and V (FP8 e4m3).

TEST INFRASTRUCTURE (see ``oracle/formats.py``): only tests, the smoke check
and the benchmark's CPU-baseline leg use this module.

What it follows.  ThriftAttention: Selective Mixed Precision for
Long-Context FP4 Attention (abstract) moves the low-precision attention
blocks to 4-bit with "block-scaled quantisation" on Blackwell; HyQuant:
Hybrid-Precision Quantization for LLM Attention (abstract) quantises "most
attention states" to low bits.  The pages give no recipe, so the standard
NVFP4 one is written out, in FP32 with correctly rounded IEEE operations
(numpy float32 arithmetic never fuses a multiply into an add):

* tensor scale per (batch, head): ``g = amax / 2688`` (2688 = 6 * 448),
  ``g = 1`` when the head is all zeros;
* per 16 consecutive elements along d: ``s = e4m3(amax_blk / (6 * g))``;
  with ``den = dec(s) * g`` every element gets ``e2m1(x / den)``; a block
  whose scale decodes to 0 gets all-zero codes;
* dequantised value: ``e2m1_dec(code) * dec(s) * g``.

V is quantised to e4m3 with one power-of-two scale per (batch, kv head,
channel): ``e_c`` is the smallest integer with ``amax_c <= 448 * 2**e_c``
(0 for an all-zero channel); ``v_code = e4m3(v * 2**-e_c)`` and the BF16
copy ``v_s = v * 2**-e_c`` feeds the BF16 tiles -- exact, except for values
that fall into the BF16 subnormals (a channel whose maximum is 2**134 or more
times larger), which round to nearest with ties to even.

Parity pins: tests/test_oracle_quantize.py (bound on the dequantisation
error, the block maximum lands on +-6, exact V rescaling, minimal e_c,
agreement with torch's own e4m3 conversion).
"""
from __future__ import annotations

import numpy as np
import torch

from .formats import e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode

F32 = np.float32


def _as_f32(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float32).numpy()
    return np.asarray(x, dtype=np.float32)


def tensor_scale(amax) -> np.ndarray:
    """Per-head tensor scale g = amax / 2688 in FP32 (1 for an all-zero head)."""
    amax = np.asarray(amax, dtype=F32)
    return np.where(amax > 0, (amax / F32(2688.0)).astype(F32), F32(1.0)).astype(F32)


def nvfp4_quantize(x, g=None):
    """NVFP4-quantise ``x[B,H,N,d]`` (BF16 values) per (B,H) head.

    ``g`` (optional, [B,H]) supplies the head's tensor scale when ``x`` holds
    only some rows of the head; by default it comes from ``x`` itself.
    Returns (codes[B,H,N,d] uint8 0..15, sf[B,H,N,d/16] uint8 e4m3 codes,
    g[B,H] float32).
    """
    x = _as_f32(x)
    B, H, N, d = x.shape
    assert d % 16 == 0
    if g is None:
        amax = np.abs(x).reshape(B, H, -1).max(axis=2) if N > 0 else np.zeros((B, H), F32)
        g = tensor_scale(amax)
    g = np.asarray(g, dtype=F32)
    blk = x.reshape(B, H, N, d // 16, 16)
    amax_b = np.abs(blk).max(axis=4)                                 # f32, exact
    six_g = (F32(6.0) * g).astype(F32)                               # f32 product
    ratio = (amax_b / six_g[:, :, None, None]).astype(F32)           # f32 quotient
    sf = e4m3_encode(ratio)
    s_dec = e4m3_decode(sf).astype(F32)                              # exact in f32
    den = (s_dec * g[:, :, None, None]).astype(F32)                  # f32 product
    safe = np.where(den > 0, den, F32(1.0)).astype(F32)
    y = (blk / safe[..., None]).astype(F32)                          # f32 quotient
    codes = e2m1_encode(y)
    codes = np.where((s_dec > 0)[..., None], codes, np.uint8(0)).astype(np.uint8)
    return codes.reshape(B, H, N, d), sf.astype(np.uint8), g


def nvfp4_dequantize(codes, sf, g) -> np.ndarray:
    """Exact float64 value of each NVFP4 element: e2m1 * dec(s) * g."""
    B, H, N, d = codes.shape
    vals = e2m1_decode(codes).reshape(B, H, N, d // 16, 16)
    s = e4m3_decode(sf)[..., None]
    out = vals * s * np.asarray(g, dtype=np.float64)[:, :, None, None, None]
    return out.reshape(B, H, N, d)


def v_channel_exponent(amax) -> np.ndarray:
    """Smallest integer e with amax <= 448 * 2**e (0 where amax == 0).

    With amax = m * 2**E (m in [0.5, 1)) and 448 = 0.875 * 2**9 the condition
    is m * 2**E <= 0.875 * 2**(9+e), i.e. e >= E - 9 when m <= 0.875 and
    e >= E - 8 otherwise: an exact integer computation.
    """
    amax = np.asarray(amax, dtype=np.float64)
    m, E = np.frexp(amax)
    e = np.where(m <= 0.875, E - 9, E - 8)
    return np.where(amax > 0, e, 0).astype(np.int64)


def fp8_v_quantize(v):
    """Quantise ``v[B,Hkv,N,d]`` to e4m3 with per-channel power-of-two scales.

    Returns (v_code[B,H,N,d] uint8 e4m3, v_exp[B,H,d] int8, v_s[B,H,N,d] float32
    holding the exact BF16 values v * 2**-e_c).
    """
    v = _as_f32(v)
    B, H, N, d = v.shape
    amax = np.abs(v).max(axis=2) if N > 0 else np.zeros((B, H, d), F32)
    e = v_channel_exponent(amax)
    # v * 2**-e_c in FP32: exact unless it falls below 2**-142, deep in the subnormals
    scaled = np.ldexp(v.astype(np.float64), (-e)[:, :, None, :].astype(np.int32)).astype(F32)
    v_code = e4m3_encode(scaled)
    # the BF16 copy: exact wherever v * 2**-e_c is a BF16 value, which every value at or
    # above 2**-126 is (8 significant bits); below, in the BF16 subnormals, round to
    # nearest, ties to even, sign kept (a value below 2**-142 rounds to +-0 either way,
    # so the FP32 rounding above cannot change the result)
    v_s = torch.from_numpy(np.ascontiguousarray(scaled)).to(torch.bfloat16).float().numpy()
    return v_code, e.astype(np.int8), v_s


def quantize(q, k, v):
    """All three quantisations, as the library's ``thrift_quantize`` computes them."""
    q_codes, q_sf, q_g = nvfp4_quantize(q)
    k_codes, k_sf, k_g = nvfp4_quantize(k)
    v_code, v_exp, v_s = fp8_v_quantize(v)
    return dict(q_codes=q_codes, q_sf=q_sf, q_g=q_g,
                k_codes=k_codes, k_sf=k_sf, k_g=k_g,
                v_code=v_code, v_exp=v_exp, v_s=v_s)


def pack_nibbles(codes) -> np.ndarray:
    """[..., d] 4-bit codes -> [..., d/2] bytes, element 2t in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out
