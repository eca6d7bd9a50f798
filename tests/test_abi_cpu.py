"""The C ABI library loads, exports every declared entry point and validates
arguments on the host (no kernel is launched: these run without a GPU)."""
import ctypes
import os
import re

import pytest

import mixed_precision_bit_quant_b200 as mq
from mixed_precision_bit_quant_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"THRIFT_API\s+[\w\s\*]+?\b(thrift_\w+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    L = mq.lib()
    names = _declared_functions()
    assert "thrift_attn_fwd" in names and "thrift_quantize" in names and "thrift_select" in names
    for n in names:
        assert hasattr(L, n), n


def test_version_and_status_strings():
    assert "sm_100a" in mq.version()
    assert mq.status_string(0) == "THRIFT_OK"
    assert mq.status_string(4) == "THRIFT_ERR_TIMEOUT"
    assert mq.launch_count() >= 0


def test_quant_and_workspace_sizes():
    s = mq.make_shape(1, 32, 8, 32768, 128, True)
    T = 256
    want = [32 * 32768 * 64, 32 * 32768 * 8, 32 * T * 2 * 512, 32 * 4,
            8 * 32768 * 64, 8 * 32768 * 8, 8 * T * 2 * 512, 8 * 4,
            8 * 128 * 32768, 8 * 128 * 32768 * 2, 8 * 128]
    assert [mq.quant_bytes(s, f) for f in range(11)] == want
    assert mq.workspace_bytes(s, mq.OP_QUANTIZE) == 4 * (32 + 8 + 8 * 128)
    assert mq.workspace_bytes(s, mq.OP_SELECT) == 4 * T * 128 * (32 + 8)
    assert mq.workspace_bytes(s, mq.OP_ATTN) == 0
    ragged = mq.make_shape(32, 12, 12, 197, 64, False)
    assert mq.quant_bytes(ragged, 8) == 32 * 12 * 64 * 256            # V^T padded to 2 tiles


@pytest.mark.parametrize("bad", [
    dict(d=96), dict(d=256),
])
def test_unsupported_head_dim(bad):
    args = dict(B=1, Hq=2, Hkv=2, N=128, d=64, causal=False)
    args.update(bad)
    s = mq.make_shape(**args)
    L = mq.lib()
    assert L.thrift_quant_bytes(ctypes.byref(s), 0) == 0
    st = L.thrift_select(ctypes.byref(s), 16, 16, 500, 0, 16, None, 16, 1 << 20, None)
    assert st == _lib.THRIFT_ERR_UNSUPPORTED


@pytest.mark.parametrize("bad", [dict(Hq=3, Hkv=2), dict(N=0), dict(B=0), dict(causal=2)])
def test_invalid_shapes_rejected_on_host(bad):
    args = dict(B=1, Hq=4, Hkv=2, N=256, d=64, causal=False)
    args.update(bad)
    s = _lib.Shape(args["B"], args["Hq"], args["Hkv"], args["N"], args["d"], args["causal"], 0.0)
    L = mq.lib()
    q = _lib.QuantStruct(*([16] * 11))
    assert L.thrift_quantize(ctypes.byref(s), 16, 16, 16, ctypes.byref(q), 16, 1 << 20, None) == _lib.THRIFT_ERR_INVALID
    assert L.thrift_attn_fwd(ctypes.byref(s), ctypes.byref(q), 16, 16, 16, 16, None, None, 0, None) == _lib.THRIFT_ERR_INVALID


def test_null_and_misaligned_pointers_rejected():
    s = mq.make_shape(1, 2, 2, 256, 64, False)
    L = mq.lib()
    q = _lib.QuantStruct(*([16] * 11))
    assert L.thrift_quantize(ctypes.byref(s), None, 16, 16, ctypes.byref(q), 16, 1 << 20, None) == 1
    assert L.thrift_quantize(ctypes.byref(s), 24, 16, 16, ctypes.byref(q), 16, 1 << 20, None) == 1
    q2 = _lib.QuantStruct(*([16] * 10 + [None]))
    assert L.thrift_attn_fwd(ctypes.byref(s), ctypes.byref(q2), 16, 16, 16, 16, None, None, 0, None) == 1
    # workspace too small
    assert L.thrift_select(ctypes.byref(s), 16, 16, 500, 0, 16, None, 16, 8, None) == 1
    # negative budget
    assert L.thrift_select(ctypes.byref(s), 16, 16, -1, 0, 16, None, 16, 1 << 20, None) == 1
    # null mask
    assert L.thrift_attn_fwd(ctypes.byref(s), ctypes.byref(q), 16, 16, None, 16, None, None, 0, None) == 1


def test_maximum_sizes_on_host():
    # the mask row of a query tile is held in shared memory: at most 4096 key tiles
    L = mq.lib()
    at_max = mq.make_shape(1, 1, 1, 4096 * 128, 128, True)
    assert L.thrift_quant_bytes(ctypes.byref(at_max), 0) == 4096 * 128 * 64
    assert L.thrift_workspace_bytes(ctypes.byref(at_max), _lib.OP_SELECT) == 4 * 4096 * 128 * 2
    over = mq.make_shape(1, 1, 1, 4096 * 128 + 1, 128, True)
    assert L.thrift_quant_bytes(ctypes.byref(over), 0) == 0
    q = _lib.QuantStruct(*([16] * 11))
    assert L.thrift_quantize(ctypes.byref(over), 16, 16, 16, ctypes.byref(q), 16, 1 << 30, None) == \
        _lib.THRIFT_ERR_UNSUPPORTED
    assert L.thrift_attn_fwd(ctypes.byref(over), ctypes.byref(q), 16, 16, 16, 16, None, None, 0, None) == \
        _lib.THRIFT_ERR_UNSUPPORTED
    # the per-head kernels put (batch, head) on grid.y: B * (Hq + Hkv) <= 65535
    wide = mq.make_shape(1, 32768, 32768, 128, 64, False)
    assert L.thrift_quant_bytes(ctypes.byref(wide), 0) == 0
    ok = mq.make_shape(1, 32767, 32767, 128, 64, False)
    assert L.thrift_quant_bytes(ctypes.byref(ok), 0) == 32767 * 128 * 32


def _dshape(B=2, Hq=8, Hkv=2, L=1000, d=128, scale=0.0):
    return _lib.DecodeShape(B, Hq, Hkv, L, d, scale)


def test_decode_cache_and_workspace_sizes():
    L = mq.lib()
    s = _dshape()
    rows = 2 * 2 * 1000
    want = [rows * 64, rows * 4, rows * 128, rows * 4]   # e2m1 K, e8m0 K scales, e4m3 V, e8m0 V scales
    assert [L.thrift_decode_cache_bytes(ctypes.byref(s), f) for f in range(4)] == want
    assert L.thrift_decode_cache_bytes(ctypes.byref(s), 4) == 0
    # one softmax state (max, sum, O[d]) per query head and 256-token chunk
    assert L.thrift_decode_workspace_bytes(ctypes.byref(s)) == 4 * 2 * 8 * 4 * (2 + 128)
    s64 = _dshape(B=1, Hq=4, Hkv=4, L=256, d=64)
    assert L.thrift_decode_cache_bytes(ctypes.byref(s64), 1) == 256 * 4 * 2
    assert L.thrift_decode_workspace_bytes(ctypes.byref(s64)) == 4 * 4 * 1 * (2 + 64)


@pytest.mark.parametrize("bad,status", [
    (dict(d=96), _lib.THRIFT_ERR_UNSUPPORTED),
    (dict(Hq=6, Hkv=2), _lib.THRIFT_ERR_UNSUPPORTED),      # group of 3 heads
    (dict(Hq=64, Hkv=2), _lib.THRIFT_ERR_UNSUPPORTED),     # group of 32 heads
    (dict(B=70000, Hq=1, Hkv=1), _lib.THRIFT_ERR_UNSUPPORTED),  # B * Hkv on one grid axis
    (dict(L=0), _lib.THRIFT_ERR_INVALID),
    (dict(Hq=6, Hkv=4), _lib.THRIFT_ERR_INVALID),
    (dict(scale=-1.0), _lib.THRIFT_ERR_INVALID),
    (dict(scale=float("inf")), _lib.THRIFT_ERR_INVALID),
])
def test_decode_shapes_rejected_on_host(bad, status):
    L = mq.lib()
    s = _dshape(**bad)
    assert L.thrift_decode_cache_bytes(ctypes.byref(s), 0) == 0
    assert L.thrift_decode_workspace_bytes(ctypes.byref(s)) == 0
    c = _lib.DecodeCacheStruct(16, 16, 16, 16)
    assert L.thrift_decode_step(ctypes.byref(s), 16, 16, 16, ctypes.byref(c), 16, None, 16, 1 << 30, None) == status
    assert L.thrift_decode_quantize_cache(ctypes.byref(s), 16, 16, ctypes.byref(c), 0, 1, None) == status


def test_decode_pointers_ranges_and_workspace_checked_on_host():
    L = mq.lib()
    s = _dshape()
    ws = L.thrift_decode_workspace_bytes(ctypes.byref(s))
    c = _lib.DecodeCacheStruct(16, 16, 16, 16)
    bad_c = _lib.DecodeCacheStruct(16, None, 16, 16)
    mis_c = _lib.DecodeCacheStruct(16, 16, 24, 16)
    step = lambda q=16, k=16, v=16, cache=c, o=16, lse=None, w=16, nb=ws: L.thrift_decode_step(  # noqa: E731
        ctypes.byref(s), q, k, v, ctypes.byref(cache), o, lse, w, nb, None)
    for kw in (dict(q=None), dict(q=24), dict(k=8), dict(o=None), dict(w=None), dict(cache=bad_c),
               dict(cache=mis_c), dict(lse=18), dict(nb=ws - 1)):
        assert step(**kw) == _lib.THRIFT_ERR_INVALID, kw
    assert L.thrift_decode_step(ctypes.byref(s), 16, 16, 16, None, 16, None, 16, ws, None) == _lib.THRIFT_ERR_INVALID
    quant = lambda t0, t1, k=16: L.thrift_decode_quantize_cache(  # noqa: E731
        ctypes.byref(s), k, 16, ctypes.byref(c), t0, t1, None)
    for t0, t1 in ((-1, 5), (0, 1001), (7, 6)):
        assert quant(t0, t1) == _lib.THRIFT_ERR_INVALID, (t0, t1)
    assert quant(0, 5, k=None) == _lib.THRIFT_ERR_INVALID
    # an empty range is valid and enqueues nothing (no device access)
    assert quant(5, 5) == _lib.THRIFT_OK
    assert quant(1000, 1000) == _lib.THRIFT_OK
