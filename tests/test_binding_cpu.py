"""Argument checks of the Python binding (no GPU: every check runs before the
library is called, and the device check is stubbed where a test needs the
others to pass on host tensors).

The C ABI reads each buffer as dense and as large as the shape implies, so the
binding refuses strided views, other dtypes, host tensors, mismatched shapes
and quantised buffers sized for a smaller problem.  The call patterns of the
benchmark and of the GPU tests are replayed here on host tensors to show they
pass every check but the device one.
"""
import pytest
import torch

import mixed_precision_bit_quant_b200 as mq
from mixed_precision_bit_quant_b200 import _lib, workloads


@pytest.fixture
def any_device(monkeypatch):
    monkeypatch.setattr(_lib, "_on_device", lambda t, name, device=None: None)


def _qkv(B=1, Hq=4, Hkv=2, N=300, d=64):
    w = workloads.custom("b", B, Hq, Hkv, N, d, True, "llm", 500, 0, seed=1)
    return workloads.generate(w)


def test_host_tensors_are_refused():
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="CUDA"):
        mq.quantize(q, k, v)
    with pytest.raises(ValueError, match="CUDA"):
        mq.select(q, k, True)


@pytest.mark.parametrize("bad", ["dtype", "strided", "shape", "rank"])
def test_bad_inputs_are_refused(any_device, bad):
    q, k, v = _qkv()
    if bad == "dtype":
        q = q.float()
    elif bad == "strided":
        k = k.transpose(2, 3).contiguous().transpose(2, 3)
    elif bad == "shape":
        v = v[:, :, :-1]
    else:
        q = q[0]
    with pytest.raises(ValueError, match={"dtype": "dtype", "strided": "contiguous", "shape": "shape",
                                          "rank": "tensor"}[bad]):
        mq.quantize(q, k, v)


def test_quantized_buffers_for_a_smaller_problem_are_refused(any_device):
    q, k, v = _qkv(N=300)
    small = mq.alloc_quantized(mq.shape_of(q[:, :, :200], k[:, :, :200], True), "cpu")
    with pytest.raises(ValueError, match="bytes"):
        _lib._check_quantized(small, mq.shape_of(q, k, True), torch.device("cpu"))


def test_output_buffers_are_checked(any_device):
    q, k, _ = _qkv()
    B, Hq, N, _ = q.shape
    T = (N + 127) // 128
    with pytest.raises(ValueError, match="mask"):
        mq.select(q, k, True, mask=torch.empty((B, Hq, T, 2), dtype=torch.int32))
    with pytest.raises(ValueError, match="counts"):
        mq.select(q, k, True, counts=torch.empty((B, Hq, T), dtype=torch.int64))
    quant = mq.alloc_quantized(mq.shape_of(q, k, True), "cpu")
    mask = torch.zeros((B, Hq, T, 1), dtype=torch.int32)
    with pytest.raises(ValueError, match="o:"):
        mq.attn_fwd(q, k, quant, mask, True, o=torch.empty_like(q, dtype=torch.float32))
    with pytest.raises(ValueError, match="lse"):
        mq.attn_fwd(q, k, quant, mask, True, lse=torch.empty((B, Hq), dtype=torch.float32))


@pytest.mark.parametrize("name", ["tiny", "vit"])
def test_benchmark_and_test_call_patterns_pass_every_check(any_device, name, monkeypatch):
    # replay the allocations bench.py and the GPU tests make, with the three compute
    # calls stubbed out: only the argument checks run
    real = _lib.lib()

    class Fake:
        def __getattr__(self, attr):
            if attr in ("thrift_quantize", "thrift_select", "thrift_attn_fwd"):
                return lambda *a: 0
            return getattr(real, attr)
    fake = Fake()
    monkeypatch.setattr(_lib, "lib", lambda: fake)
    monkeypatch.setattr(_lib, "_stream", lambda: 0)
    w = workloads.WORKLOADS[name]
    q, k, v = workloads.generate(w)
    shape = mq.shape_of(q, k, w.causal)
    quant = mq.alloc_quantized(shape, "cpu")
    ws_q = torch.empty(max(16, mq.workspace_bytes(shape, mq.OP_QUANTIZE)), dtype=torch.uint8)
    ws_s = torch.empty(max(16, mq.workspace_bytes(shape, mq.OP_SELECT)), dtype=torch.uint8)
    T, W = w.T, (w.T + 31) // 32
    mask = torch.empty((w.B, w.Hq, T, W), dtype=torch.int32)
    counts = torch.empty((w.B, w.Hq, T), dtype=torch.int32)
    o = torch.empty_like(q)
    mq.quantize(q, k, v, w.causal, out=quant, ws=ws_q)
    mq.select(q, k, w.causal, w.budget_bp, w.budget_tiles, mask=mask, counts=counts, ws=ws_s)
    mq.attn_fwd(q, k, quant, mask, w.causal, o=o)
    # the defaults the GPU tests and smoke() use
    quant2 = mq.quantize(q, k, v)
    mask2, _ = mq.select(q, k, w.causal, w.budget_bp, w.budget_tiles)
    o2, lse2 = mq.attn_fwd(q, k, quant2, mask2, w.causal, want_lse=True)
    assert o2.shape == q.shape and lse2.shape == q.shape[:3]
    # the second buffer set of the end-to-end leg
    qb, kb, vb, ob = (torch.empty_like(t) for t in (q, k, v, o))
    mq.quantize(qb, kb, vb, w.causal, out=quant, ws=ws_q)
    mq.attn_fwd(qb, kb, quant, mask, w.causal, o=ob)


def _decode_inputs(B=2, Hq=8, Hkv=2, L=300, d=64):
    g = torch.Generator().manual_seed(5)
    q = torch.randn((B, Hq, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, L, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, L, d), generator=g).to(torch.bfloat16)
    return q, k, v


def _host_cache(k):
    B, Hkv, L, d = k.shape
    rows = B * Hkv * L
    sizes = dict(kc=rows * d // 2, ksc=rows * d // 32, vc=rows * d, vsc=rows * d // 32)
    return {f: torch.zeros(n, dtype=torch.uint8) for f, n in sizes.items()}


def test_decode_host_tensors_are_refused():
    q, k, v = _decode_inputs()
    with pytest.raises(ValueError, match="CUDA"):
        mq.decode_quantize_cache(k, v)
    with pytest.raises(ValueError, match="CUDA"):
        mq.decode_step(q, k, v, _host_cache(k))


@pytest.mark.parametrize("bad", ["k_dtype", "v_shape", "q_rank", "q_batch", "q_dim", "cache_small",
                                 "cache_dtype", "o_dtype", "lse_shape", "strided_v"])
def test_decode_bad_arguments_are_refused(any_device, bad):
    q, k, v = _decode_inputs()
    cache = _host_cache(k)
    kw = {}
    match = {"k_dtype": "dtype", "v_shape": "shape", "q_rank": "tensor", "q_batch": "shape", "q_dim": "shape",
             "cache_small": "too small", "cache_dtype": "dtype", "o_dtype": "dtype", "lse_shape": "shape",
             "strided_v": "contiguous"}[bad]
    if bad == "k_dtype":
        k = k.float()
    elif bad == "v_shape":
        v = v[:, :, :-1]
    elif bad == "q_rank":
        q = q[0]
    elif bad == "q_batch":
        q = q[:1]
    elif bad == "q_dim":
        q = torch.zeros((2, 8, 128), dtype=torch.bfloat16)
    elif bad == "cache_small":
        cache["vc"] = cache["vc"][:-1]
    elif bad == "cache_dtype":
        cache["ksc"] = cache["ksc"].to(torch.int32)
    elif bad == "o_dtype":
        kw["o"] = torch.empty(q.shape, dtype=torch.float32)
    elif bad == "lse_shape":
        kw["lse"] = torch.empty((2, 7), dtype=torch.float32)
    else:
        v = v.transpose(2, 3).contiguous().transpose(2, 3)
    with pytest.raises(ValueError, match=match):
        mq.decode_step(q, k, v, cache, **kw)
