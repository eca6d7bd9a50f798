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
