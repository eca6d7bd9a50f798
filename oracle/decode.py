"""Oracle: one decode step against a mixed-precision KV cache (FP64).

TEST INFRASTRUCTURE (see ``oracle/formats.py``): only tests, the smoke check
and the benchmark's CPU-baseline leg use this module.

What it follows.  HyQuant: Hybrid-Precision Quantization for LLM Attention
(abstract, decode stage) compresses the KV cache with the principle of its
prefill operator -- sink ("vertical-line") tokens and the local window stay in
high precision, the rest is low-bit -- and fuses the dequantisation into the
attention.  The page gives no formats or sizes, so this library fixes them:

* the cache grows one token at a time, so every token is quantised on its own
  (no per-head tensor scale that would change as the cache grows): K as MXFP4
  and V as MXFP8 (e4m3), each with one e8m0 scale per 32 channels of the
  token (``oracle.mx``);
* high precision (BF16, as stored) for the sink tile -- tokens [0, 128) -- and
  the local window -- the last 128 tokens [L - 128, L); every other token is
  read from its quantised form;
* the query of the step stays BF16 (decode is bound by reading the cache, so
  there is no low-bit query product to gain);
* query head h reads kv head h // (Hq / Hkv); logits q . k_t / sqrt(d); exact
  softmax over all L tokens (P is not rounded); output sum_t p_t v_t and
  LSE = max + ln(sum).

Parity pins: tests/test_oracle_decode.py.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from . import mx

SINK = 128
WINDOW = 128


def _f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def quantize_cache(k, v):
    """Per-token MX quantisation of a cache ``k, v[B,Hkv,L,d]`` (blocks of 32 along d)."""
    k_codes, k_sc = mx.mx_quantize(k, "e2m1", axis=3)
    v_codes, v_sc = mx.mx_quantize(v, "e4m3", axis=3)
    return dict(k_codes=k_codes, k_sc=k_sc, v_codes=v_codes, v_sc=v_sc)


def high_precision_tokens(L: int) -> np.ndarray:
    """Boolean [L]: the sink tile and the local window."""
    t = np.arange(L)
    return (t < SINK) | (t >= L - WINDOW)


def cache_views(k, v, cache):
    """FP64 (K', V') the decode step reads: BF16 rows for sink and window, dequantised rows elsewhere."""
    k_hi, v_hi = _f64(k), _f64(v)
    k_lo = mx.mx_dequantize(cache["k_codes"], cache["k_sc"], "e2m1", axis=3)
    v_lo = mx.mx_dequantize(cache["v_codes"], cache["v_sc"], "e4m3", axis=3)
    hp = high_precision_tokens(k_hi.shape[2])[None, None, :, None]
    return np.where(hp, k_hi, k_lo), np.where(hp, v_hi, v_lo)


def decode_step(q, k, v, cache=None, sm_scale: float = 0.0):
    """One decode step: ``q[B,Hq,d]`` against the cache ``k, v[B,Hkv,L,d]``.

    ``cache``: the quantised cache (``quantize_cache``), or None to build it.
    Returns (o[B,Hq,d] float64, lse[B,Hq] float64).
    """
    q = _f64(q)
    B, Hq, d = q.shape
    Hkv, L = int(k.shape[1]), int(k.shape[2])
    G = Hq // Hkv
    scale = sm_scale if sm_scale > 0 else 1.0 / math.sqrt(d)
    kk, vv = cache_views(k, v, cache if cache is not None else quantize_cache(k, v))
    o = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hq):
            s = (kk[b, h // G] @ q[b, h]) * scale
            m = s.max()
            p = np.exp(s - m)
            o[b, h] = (p @ vv[b, h // G]) / p.sum()
            lse[b, h] = m + math.log(p.sum())
    return o, lse
