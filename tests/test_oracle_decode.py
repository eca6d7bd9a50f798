"""Pins of the decode-step oracle (oracle/decode.py).

Closed forms and invariants the definition fixes: a cache that is all sink and
window is plain softmax attention over the BF16 cache; otherwise the step is
softmax attention over the cache as read (BF16 rows where kept, dequantised MX
rows elsewhere), computed here independently with one einsum per batch;
per-token quantisation makes the cache appendable (quantising token by token
equals quantising the whole cache); a constant V gives that constant; a zero
query gives the mean of the rows read; and the rows that are read in high
precision are exactly the first and last 128.
"""
import math

import numpy as np
import pytest
import torch

from oracle import decode as odec
from oracle import mx


def _inputs(B, Hq, Hkv, L, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    k = (torch.randn(B, Hkv, L, d, generator=g) * 2).to(torch.bfloat16)
    v = torch.randn(B, Hkv, L, d, generator=g).to(torch.bfloat16)
    return q, k, v


def _softmax_attention(q, K, V, G, scale):
    # q[B,Hq,d], K/V[B,Hkv,L,d] float64 -> o[B,Hq,d]
    Kq = np.repeat(K, G, axis=1)
    Vq = np.repeat(V, G, axis=1)
    s = np.einsum("bhd,bhld->bhl", q, Kq) * scale
    s -= s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=-1, keepdims=True)
    return np.einsum("bhl,bhld->bhd", p, Vq)


@pytest.mark.parametrize("L", [1, 100, 256])
def test_short_cache_is_softmax_attention_over_bf16(L):
    q, k, v = _inputs(1, 4, 2, L, 64, 1)
    o, _ = odec.decode_step(q, k, v)
    ref = _softmax_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), 2, 1 / 8)
    assert np.abs(o - ref).max() < 1e-12


@pytest.mark.parametrize("L,d", [(257, 64), (700, 128)])
def test_long_cache_is_softmax_attention_over_the_rows_read(L, d):
    q, k, v = _inputs(2, 4, 1, L, d, 2)
    cache = odec.quantize_cache(k, v)
    o, lse = odec.decode_step(q, k, v, cache)
    kd = mx.mx_dequantize(cache["k_codes"], cache["k_sc"], "e2m1", axis=3)
    vd = mx.mx_dequantize(cache["v_codes"], cache["v_sc"], "e4m3", axis=3)
    K, V = kd.copy(), vd.copy()
    K[:, :, :128] = k[:, :, :128].double().numpy()
    V[:, :, :128] = v[:, :, :128].double().numpy()
    K[:, :, L - 128:] = k[:, :, L - 128:].double().numpy()
    V[:, :, L - 128:] = v[:, :, L - 128:].double().numpy()
    ref = _softmax_attention(q.double().numpy(), K, V, 4, 1 / math.sqrt(d))
    assert np.abs(o - ref).max() < 1e-12
    # and the quantised rows really differ from BF16 somewhere in the middle
    assert not np.array_equal(kd[:, :, 128:L - 128], k[:, :, 128:L - 128].double().numpy())


def test_cache_is_appendable_token_by_token():
    _, k, v = _inputs(1, 1, 2, 40, 64, 3)
    whole = odec.quantize_cache(k, v)
    for t in range(40):
        one = odec.quantize_cache(k[:, :, t:t + 1], v[:, :, t:t + 1])
        for f in whole:
            assert np.array_equal(one[f][:, :, 0], whole[f][:, :, t]), (f, t)


def test_constant_values_and_zero_query():
    q, k, v = _inputs(1, 2, 1, 500, 64, 4)
    vc = torch.full_like(v, 0.75)
    o, _ = odec.decode_step(q, k, vc)
    assert np.abs(o - 0.75).max() < 1e-12            # 0.75 is exact in e4m3
    oz, lse = odec.decode_step(torch.zeros_like(q), k, v)
    K, V = odec.cache_views(k, v, odec.quantize_cache(k, v))
    assert np.abs(oz - V.mean(axis=2)[:, [0, 0]]).max() < 1e-12
    assert np.allclose(lse, math.log(500))


def test_high_precision_rows_are_sink_and_window():
    for L in (1, 128, 129, 256, 257, 1000):
        hp = odec.high_precision_tokens(L)
        want = [t < 128 or t >= L - 128 for t in range(L)]
        assert hp.tolist() == want
