"""GPU parity of the decode step against a mixed-precision KV cache
(thrift_decode_quantize_cache, thrift_decode_step) and the oracle
(oracle/decode.py; HyQuant: Hybrid-Precision Quantization for LLM Attention,
abstract, decode stage).

Bar: the cache's e2m1 / e4m3 codes and e8m0 scales bit-exact, appending
tokens one at a time equal to quantising the whole cache, and the output
within max|err| <= 2e-2 * max|O_ref| and relative L2 <= 5e-3 (LSE within
1e-3) of the oracle on the same seeded inputs.
"""
import math

import numpy as np
import pytest
import torch

import mixed_precision_bit_quant_b200 as mq
from oracle import decode as odec

pytestmark = pytest.mark.gpu


def _inputs(B, Hq, Hkv, L, d, seed):
    """Decode-shaped inputs: the llm workloads' generator for the cache (K ~ N(0,1) plus a
    per-(kv head, channel) offset of standard deviation 2, token 0 scaled by 8 as a sink;
    V ~ N(0,1)) and one BF16 query per sequence and head."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, d), generator=g)
    k = torch.randn((B, Hkv, L, d), generator=g) + 2.0 * torch.randn((B, Hkv, 1, d), generator=g)
    k[:, :, 0, :] *= 8.0
    v = torch.randn((B, Hkv, L, d), generator=g)
    return tuple(t.to(torch.bfloat16).contiguous() for t in (q, k, v))


def _check_cache(k, v, cache):
    B, Hkv, L, d = k.shape
    ref = odec.quantize_cache(k, v)
    got = {f: t.cpu().numpy() for f, t in cache.items()}
    kc = ref["k_codes"].reshape(B, Hkv, L, d // 2, 2)
    packed = (kc[..., 0] | (kc[..., 1] << 4)).astype(np.uint8)
    assert np.array_equal(got["kc"].reshape(packed.shape), packed), "K codes"
    assert np.array_equal(got["ksc"].reshape(ref["k_sc"].shape), ref["k_sc"]), "K scales"
    assert np.array_equal(got["vc"].reshape(ref["v_codes"].shape), ref["v_codes"]), "V codes"
    assert np.array_equal(got["vsc"].reshape(ref["v_sc"].shape), ref["v_sc"]), "V scales"


def _run(B, Hq, Hkv, L, d, seed=0, scale=0.0, check_cache=True, batches=None, q_mul=1.0):
    q, k, v = _inputs(B, Hq, Hkv, L, d, seed)
    if q_mul != 1.0:  # a power of two: the BF16 query is scaled exactly
        q = (q.float() * q_mul).to(torch.bfloat16)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    cache = mq.decode_quantize_cache(kd, vd)
    o, lse = mq.decode_step(qd, kd, vd, cache, softmax_scale=scale, want_lse=True)
    st, word = mq.device_status()
    assert st == 0, f"device watchdog raised {word:#x}"
    if check_cache:
        _check_cache(k, v, cache)
    for b in (range(B) if batches is None else batches):
        o_ref, lse_ref = odec.decode_step(q[b:b + 1], k[b:b + 1], v[b:b + 1], sm_scale=scale)
        og = o[b:b + 1].float().cpu().numpy().astype(np.float64)
        err = np.abs(og - o_ref).max() / np.abs(o_ref).max()
        rel = np.linalg.norm(og - o_ref) / np.linalg.norm(o_ref)
        assert err <= 2e-2 and rel <= 5e-3, (b, err, rel)
        assert np.abs(lse[b:b + 1].cpu().numpy() - lse_ref).max() < 1e-3


@pytest.mark.parametrize("B,Hq,Hkv,L,d", [
    (1, 4, 2, 1, 64),          # one token (sink only)
    (2, 4, 4, 100, 128),       # all sink / window
    (1, 8, 2, 256, 128),       # sink + window exactly
    (2, 8, 2, 257, 64),        # one quantised token
    (1, 16, 1, 700, 128),      # G = 16 (the largest group)
    (3, 32, 8, 1000, 128),     # ragged last chunk
    (1, 4, 4, 4096, 64),
])
def test_decode_shapes(B, Hq, Hkv, L, d):
    _run(B, Hq, Hkv, L, d, seed=L + d)


def test_decode_llm32k_cache():
    """The llm shape (Hq 32, Hkv 8, d 128) with a 32K-token cache."""
    _run(1, 32, 8, 32768, 128, seed=1, check_cache=False)


def test_decode_benchmark_shape_sampled_batches():
    """The benchmark's decode workload (B 8, 32K-token caches), two batches checked."""
    _run(8, 32, 8, 32768, 128, seed=2, check_cache=False, batches=[0, 7])


def test_decode_custom_scale():
    _run(2, 8, 2, 900, 128, seed=5, scale=0.2)


def test_decode_cache_is_appendable():
    q, k, v = _inputs(2, 8, 2, 300, 128, 7)
    kd, vd = k.cuda(), v.cuda()
    whole = mq.decode_quantize_cache(kd, vd)
    part = mq.decode_quantize_cache(kd, vd, t_end=200)
    for t in range(200, 300, 7):
        mq.decode_quantize_cache(kd, vd, cache=part, t_begin=t, t_end=min(300, t + 7))
    torch.cuda.synchronize()
    for f in whole:
        assert torch.equal(whole[f], part[f]), f


@pytest.mark.parametrize("q_mul,scale", [(2.0 ** -24, 2.0 ** 24), (2.0 ** 12, 2.0 ** -12)])
def test_decode_query_magnitude_extremes(q_mul, scale):
    """The logits of quantised tokens run in FP16 with the query rescaled per head by a
    power of two; a query 2^24 times smaller or 2^12 times larger than usual (softmax
    scale compensating, so the logits are the usual ones) must still match the oracle."""
    _run(2, 8, 2, 1024, 128, seed=11, scale=scale / math.sqrt(128), check_cache=False, q_mul=q_mul)
