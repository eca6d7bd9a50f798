"""Oracle: microscaling (MX) formats, the MXFP4 / MXFP8 variant of the low path.

TEST INFRASTRUCTURE (see ``oracle/formats.py``): only tests, the smoke check
and the benchmark's CPU-baseline leg use this module.

What it follows.  The attention-quantization topic page lists MXFP4 next to
NVFP4 among the block-scaled 4-bit formats (its paper list: "Bridging the Gap
Between Promise and Performance for Microscaling FP4 Quantization", "MicroMix",
and "Diagonal-Tiled Mixed-Precision Attention for Efficient Low-Bit MXFP
Inference").  The pages print no definition, so the standard one (the OCP
Microscaling Formats specification, v1.0) is written out:

* a block is 32 consecutive elements; it shares one scale X = 2**e stored as
  an e8m0 code (unsigned, bias 127, code 255 is NaN, no zero);
* e = floor(log2(amax_block)) - emax_elem, where emax_elem is the exponent of
  the element format's largest normal value (2 for e2m1, whose largest value
  is 6 = 1.5 * 2**2; 8 for e4m3, 448 = 1.75 * 2**8), clamped to [-127, 127];
* every element becomes elem(x / X), rounded to nearest with ties to the even
  code and saturated at the element format's largest value (the same roundings
  as ``oracle.formats``);
* the dequantised value is elem_dec(code) * X.

Because e is taken from the block maximum's binade alone, a block maximum whose
mantissa exceeds the element format's largest one (1.5 for e2m1, 1.75 for
e4m3) saturates to the largest element value: amax / X lies in [4, 8) for
e2m1 and in [256, 512) for e4m3.  That is the specification's behaviour and
is kept.

Readings where the specification leaves a choice: an all-zero block takes
e = -127 (code 0) and zero codes; the sign of zero is kept as in the NVFP4
path.  For the attention variant, Q and K are MXFP4 with blocks along d; V is
MXFP8 (e4m3) with blocks of 32 keys along N for each channel, because the
P.V contraction runs over keys; a ragged last block holds only the valid keys
(the missing ones count as zeros, which never raise the block maximum).

Every operation below is exact: x / X with X a power of two is a scaling by
2**-e, done with ``np.ldexp`` in float64.

Parity pins: tests/test_oracle_mx.py.
"""
from __future__ import annotations

import numpy as np
import torch

from .formats import e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode

MX_BLOCK = 32
EMAX_E2M1 = 2
EMAX_E4M3 = 8


def _f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def e8m0_decode(codes) -> np.ndarray:
    """e8m0 scale codes (0..255) -> float64 2**(code - 127); NaN for 255."""
    c = np.asarray(codes).astype(np.int64)
    return np.where(c == 255, np.nan, np.ldexp(1.0, c - 127))


def mx_shared_exponent(amax, emax_elem: int) -> np.ndarray:
    """e = floor(log2(amax)) - emax_elem, clamped to [-127, 127]; -127 for amax == 0.

    With amax = m * 2**E, m in [0.5, 1) (numpy's frexp), floor(log2(amax)) = E - 1
    exactly, subnormal inputs included.
    """
    amax = np.asarray(amax, dtype=np.float64)
    _, E = np.frexp(amax)
    e = (E.astype(np.int64) - 1) - emax_elem
    e = np.clip(e, -127, 127)
    return np.where(amax > 0, e, -127).astype(np.int64)


def _blocks(x, axis: int):
    """Move ``axis`` last and split it into blocks of 32 (zero padded)."""
    x = np.moveaxis(_f64(x), axis, -1)
    n = x.shape[-1]
    nb = (n + MX_BLOCK - 1) // MX_BLOCK
    pad = nb * MX_BLOCK - n
    if pad:
        x = np.concatenate([x, np.zeros(x.shape[:-1] + (pad,))], axis=-1)
    return x.reshape(x.shape[:-1] + (nb, MX_BLOCK)), n


def _unblocks(xb, n: int, axis: int):
    x = xb.reshape(xb.shape[:-2] + (-1,))[..., :n]
    return np.moveaxis(x, -1, axis)


def mx_quantize(x, elem: str, axis: int = -1):
    """MX-quantise ``x`` with blocks of 32 along ``axis``.

    ``elem``: "e2m1" (MXFP4) or "e4m3" (MXFP8).  Returns (codes, scale codes):
    codes has the shape of ``x`` (uint8: 4-bit e2m1 codes or e4m3 bytes), the
    scale codes have ``axis`` replaced by the block count (uint8 e8m0).
    """
    enc, emax = (e2m1_encode, EMAX_E2M1) if elem == "e2m1" else (e4m3_encode, EMAX_E4M3)
    xb, n = _blocks(x, axis)
    e = mx_shared_exponent(np.abs(xb).max(axis=-1), emax)
    y = np.ldexp(xb, (-e)[..., None])                      # x / 2**e, exact
    codes = enc(y)
    codes = _unblocks(codes, n, axis).astype(np.uint8)
    scales = np.moveaxis((e + 127).astype(np.uint8), -1, axis)
    return codes, scales


def mx_dequantize(codes, scales, elem: str, axis: int = -1) -> np.ndarray:
    """Exact float64 values elem_dec(code) * 2**(scale - 127)."""
    dec = e2m1_decode if elem == "e2m1" else e4m3_decode
    vals = dec(codes)
    vb, n = _blocks(vals, axis)
    s = e8m0_decode(np.moveaxis(np.asarray(scales), axis, -1))
    return _unblocks(vb * s[..., None], n, axis)


def quantize(q, k, v):
    """The MX variant of the three quantisations: MXFP4 Q, K along d; MXFP8 V along N."""
    q_codes, q_sc = mx_quantize(q, "e2m1", axis=3)
    k_codes, k_sc = mx_quantize(k, "e2m1", axis=3)
    v_codes, v_sc = mx_quantize(v, "e4m3", axis=2)
    return dict(q_codes=q_codes, q_sc=q_sc, k_codes=k_codes, k_sc=k_sc, v_codes=v_codes, v_sc=v_sc)


def dequantized(quant):
    """FP64 (q_hat, k_hat, v_hat) of an MX-quantised problem."""
    return (mx_dequantize(quant["q_codes"], quant["q_sc"], "e2m1", axis=3),
            mx_dequantize(quant["k_codes"], quant["k_sc"], "e2m1", axis=3),
            mx_dequantize(quant["v_codes"], quant["v_sc"], "e4m3", axis=2))
