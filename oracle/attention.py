"""Oracle: mixed FP4/BF16 tiled attention with one online softmax (FP64).

TEST INFRASTRUCTURE (see ``oracle/formats.py``): only tests, the smoke check
and the benchmark's CPU-baseline leg use this module.

What it follows.  ThriftAttention: Selective Mixed Precision for
Long-Context FP4 Attention (abstract, second stage): the selected blocks are
computed in high precision, the rest in FP4, and both paths are merged by
online softmax into a single output.  HyQuant: Hybrid-Precision Quantization
for LLM Attention (abstract) does the same in prefill with one
hybrid-precision operator.  Written out, for every (batch b, query head h,
query tile i) and the key tiles j of C_i in ascending order:

* FP4 tile:  S = (Qhat_i . Khat_j^T) / sqrt(d) with the dequantised NVFP4
  values; BF16 tile: S = (Q_i . K_j^T) / sqrt(d) with the BF16 inputs;
* causal (key index > query index) and ragged (key index >= N) entries are
  -inf;
* exact running maximum m' = max(m, rowmax S) (no lazy rescaling),
  p = exp(S - m'), l <- l * exp(m - m') + sum p (uncast p);
* O <- O * exp(m - m') + c(p) . V'_j where, on FP4 tiles, c(p) =
  e4m3(p * 2**sigma) * 2**-sigma and V' = dec(v_code) * 2**e_c, and on BF16
  tiles c(p) = bf16(p * 2**sigma) * 2**-sigma and V' = V;
* output O / l and LSE = m + ln l.

``p_cast=False`` switches c(p) to the identity; the pins use it to reduce
the method to plain softmax attention.  Query head h reads kv head
h // (Hq / Hkv).  sigma = 8 keeps p down to e**-12.5 representable in e4m3
(the literal reading, sigma = 0, is available as a parameter).

Parity pins: tests/test_oracle_attention.py (all-BF16 budget equals exact
softmax attention, zero budget equals attention on the dequantised inputs,
probability rows sum to one, constant V and zero Q closed forms, the
single-key case).
"""
from __future__ import annotations

import math

import numpy as np
import torch

from . import mx
from .formats import bf16_round, e4m3_decode, e4m3_encode
from .quantize import fp8_v_quantize, nvfp4_dequantize, nvfp4_quantize, tensor_scale
from .select import mask_bit


def _f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


class Operands:
    """The FP64 views of one problem that the tile loop reads, built per head on demand.

    ``quant`` may hold the full quantised operands (as ``oracle.quantize.quantize``
    returns them); when it is None each head is quantised when first needed,
    with the same per-head arithmetic (query tiles use the head's tensor scale
    from the whole head and quantise only their own rows).

    ``fmt = "mx"`` takes the low path's operands from the microscaling variant
    instead (``oracle.mx``: MXFP4 Q and K, MXFP8 V; ``quant`` then holds what
    ``oracle.mx.quantize`` returns, or None to quantise the whole problem);
    ``fmt = "mxfp4_qk"`` takes MXFP4 Q and K but keeps V's per-channel FP8
    (``quant`` is then None).
    """

    def __init__(self, q, k, v, quant, causal: bool, sm_scale: float = 0.0, fmt: str = "nvfp4"):
        self._q, self._k, self._v = q, k, v
        self.quant = quant
        self.B, self.Hq, self.N, self.d = tuple(q.shape)
        self.Hkv = int(k.shape[1])
        self.G = self.Hq // self.Hkv
        self.T = (self.N + 127) // 128
        self.causal = causal
        self.sm_scale = sm_scale if sm_scale > 0 else 1.0 / math.sqrt(self.d)
        self._qc = {}
        self._kc = {}
        self.fmt = fmt
        if fmt == "mx":
            self._mx = mx.dequantized(quant if quant is not None else mx.quantize(q, k, v))
        elif fmt == "mxfp4_qk":
            qh, kh, _ = mx.dequantized(mx.quantize(q, k, v))
            v_code, v_exp, _ = fp8_v_quantize(v)
            vh = e4m3_decode(v_code) * np.ldexp(1.0, np.asarray(v_exp, dtype=np.int64))[:, :, None, :]
            self._mx = (qh, kh, vh)
        elif fmt != "nvfp4":
            raise ValueError(fmt)

    def q_tile(self, b: int, h: int, r0: int, r1: int):
        qz = self.quant
        q_hi = _f64(self._q[b, h, r0:r1])
        if self.fmt != "nvfp4":
            q_lo = self._mx[0][b, h, r0:r1]
        elif qz is not None:
            q_lo = nvfp4_dequantize(qz["q_codes"][b:b + 1, h:h + 1, r0:r1], qz["q_sf"][b:b + 1, h:h + 1, r0:r1],
                                    np.asarray(qz["q_g"])[b:b + 1, h:h + 1])[0, 0]
        else:
            key = (b, h)
            if key not in self._qc:
                head = self._q[b, h]
                amax = float(head.abs().max()) if isinstance(head, torch.Tensor) else float(np.abs(head).max())
                self._qc = {key: tensor_scale(np.array([[amax]], dtype=np.float32))}
            g = self._qc[key]
            rows = self._q[b:b + 1, h:h + 1, r0:r1]
            codes, sf, g = nvfp4_quantize(rows, g=g)
            q_lo = nvfp4_dequantize(codes, sf, g)[0, 0]
        return q_hi, q_lo

    def kv_views(self, b: int, hk: int):
        key = (b, hk)
        if self.fmt != "nvfp4":
            return _f64(self._k[b, hk]), self._mx[1][b, hk], _f64(self._v[b, hk]), self._mx[2][b, hk]
        if key not in self._kc:
            qz = self.quant
            if qz is None:
                codes, sf, g = nvfp4_quantize(self._k[b:b + 1, hk:hk + 1])
                v_code, v_exp, _ = fp8_v_quantize(self._v[b:b + 1, hk:hk + 1])
                qz = dict(k_codes=codes, k_sf=sf, k_g=g, v_code=v_code, v_exp=v_exp)
                bb, hh = 0, 0
            else:
                bb, hh = b, hk
            k_hi = _f64(self._k[b, hk])
            k_lo = nvfp4_dequantize(qz["k_codes"][bb:bb + 1, hh:hh + 1], qz["k_sf"][bb:bb + 1, hh:hh + 1],
                                    np.asarray(qz["k_g"])[bb:bb + 1, hh:hh + 1])[0, 0]
            v_hi = _f64(self._v[b, hk])
            e = np.asarray(qz["v_exp"], dtype=np.int64)[bb, hh]
            v_lo = e4m3_decode(qz["v_code"][bb, hh]) * np.ldexp(1.0, e)[None, :]
            self._kc = {key: (k_hi, k_lo, v_hi, v_lo)}
        return self._kc[key]


def attn_query_tile(ops: Operands, mask, b: int, h: int, i: int,
                    sigma: int = 8, p_cast: bool = True):
    """Rows [128 i, 128 i + 128) of the output for (b, h): returns (O[rows,d], lse[rows])."""
    hk = h // ops.G
    r0 = i * 128
    r1 = min(ops.N, r0 + 128)
    rows = np.arange(r0, r1)
    nr = r1 - r0
    q_hi, q_lo = ops.q_tile(b, h, r0, r1)
    k_hi, k_lo, v_hi, v_lo = ops.kv_views(b, hk)
    m = np.full(nr, -np.inf)
    l = np.zeros(nr)
    O = np.zeros((nr, ops.d))
    up = 2.0 ** sigma
    n_tiles = i + 1 if ops.causal else ops.T
    for j in range(n_tiles):
        c0 = j * 128
        c1 = min(ops.N, c0 + 128)
        cols = np.arange(c0, c1)
        hi = mask_bit(mask, b, h, i, j)
        if hi:
            S = (q_hi @ k_hi[c0:c1].T) * ops.sm_scale
            Vp = v_hi[c0:c1]
        else:
            S = (q_lo @ k_lo[c0:c1].T) * ops.sm_scale
            Vp = v_lo[c0:c1]
        if ops.causal:
            S = np.where(cols[None, :] > rows[:, None], -np.inf, S)
        m_new = np.maximum(m, S.max(axis=1))
        alpha = np.where(np.isneginf(m), 0.0, np.exp(m - np.where(np.isneginf(m_new), 0.0, m_new)))
        p = np.exp(S - m_new[:, None])
        l = l * alpha + p.sum(axis=1)
        if p_cast:
            if hi:
                cp = bf16_round(p * up) / up
            else:
                cp = e4m3_decode(e4m3_encode(p * up)) / up
        else:
            cp = p
        O = O * alpha[:, None] + cp @ Vp
        m = m_new
    out = O / l[:, None]
    lse = m + np.log(l)
    return out, lse


def attn_forward(q, k, v, quant, mask, causal: bool, sm_scale: float = 0.0,
                 sigma: int = 8, p_cast: bool = True, tiles=None, fmt: str = "nvfp4"):
    """Full (or sampled) mixed-precision attention forward.

    ``quant``: the quantised operands, or None to quantise each head on demand.

    ``tiles``: optional list of (b, h, i) query tiles; when given only those
    rows of the output are filled (the rest stay NaN).
    Returns (O[B,Hq,N,d] float64, lse[B,Hq,N] float64).
    """
    ops = Operands(q, k, v, quant, causal, sm_scale, fmt)
    O = np.full((ops.B, ops.Hq, ops.N, ops.d), np.nan)
    lse = np.full((ops.B, ops.Hq, ops.N), np.nan)
    if tiles is None:
        tiles = [(b, h, i) for b in range(ops.B) for h in range(ops.Hq) for i in range(ops.T)]
    for (b, h, i) in tiles:
        o, s = attn_query_tile(ops, mask, b, h, i, sigma, p_cast)
        r0 = i * 128
        O[b, h, r0:r0 + o.shape[0]] = o
        lse[b, h, r0:r0 + o.shape[0]] = s
    return O, lse


def exact_attention(q, k, v, causal: bool, sm_scale: float = 0.0):
    """Textbook one-pass softmax attention in FP64 (no tiles, no quantisation)."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, Hq, N, d = q.shape
    G = Hq // k.shape[1]
    scale = sm_scale if sm_scale > 0 else 1.0 / math.sqrt(d)
    kk = np.repeat(k, G, axis=1)
    vv = np.repeat(v, G, axis=1)
    S = np.einsum("bhnd,bhmd->bhnm", q, kk) * scale
    if causal:
        S = np.where(np.tril(np.ones((N, N), dtype=bool)), S, -np.inf)
    S = S - S.max(axis=-1, keepdims=True)
    P = np.exp(S)
    P = P / P.sum(axis=-1, keepdims=True)
    return np.einsum("bhnm,bhmd->bhnd", P, vv)


def exact_attention_tiles(q, k, v, causal: bool, tiles, sm_scale: float = 0.0):
    """Textbook softmax attention in FP64 for the rows of the given query tiles.

    The same definition as ``exact_attention`` (no tiles, no quantisation,
    one softmax per row over every visible key), restricted to the rows
    [128 i, 128 i + 128) of each (b, h, i) in ``tiles`` so that long
    sequences do not need the whole N x N logit matrix.  Rows outside the
    listed tiles stay NaN.  Returns O[B, Hq, N, d] float64.
    """
    B, Hq, N, d = tuple(q.shape)
    G = Hq // int(k.shape[1])
    scale = sm_scale if sm_scale > 0 else 1.0 / math.sqrt(d)
    O = np.full((B, Hq, N, d), np.nan)
    for (b, h, i) in tiles:
        r0, r1 = i * 128, min(N, (i + 1) * 128)
        n_keys = r1 if causal else N
        qr = _f64(q[b, h, r0:r1])
        kk = _f64(k[b, h // G, :n_keys])
        vv = _f64(v[b, h // G, :n_keys])
        S = (qr @ kk.T) * scale
        if causal:
            rows = np.arange(r0, r1)[:, None]
            S = np.where(np.arange(n_keys)[None, :] > rows, -np.inf, S)
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        O[b, h, r0:r1] = (P / P.sum(axis=1, keepdims=True)) @ vv
    return O
