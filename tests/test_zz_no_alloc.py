"""thrift_quantize_noalloc against thrift_quantize.

Some callers cannot give the library a device workspace: a C host program
that owns only its input and output buffers, code running in a host callback
or an allocator hook where allocating is not allowed, or a process whose
device memory pool belongs to another component.  For them the library keeps
the quantiser's amax scratch in a fixed device array.  This test calls that
entry point through the C ABI twice in a row (the second call reuses the
scratch the first one left behind, with smaller inputs, so stale contents
would show) and requires results identical to the workspace call.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixed_precision_bit_quant_b200 as mq
from mixed_precision_bit_quant_b200 import _lib, workloads

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    f = mq.lib().thrift_quantize_noalloc
    f.argtypes = [ctypes.POINTER(_lib.Shape), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.POINTER(_lib.QuantStruct), ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def _quantize_noalloc(q, k, v, out):
    shape = mq.shape_of(q, k, True)
    st = out.struct()
    return _noalloc_fn()(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(st),
                         torch.cuda.current_stream().cuda_stream)


def _inputs(scale, seed):
    w = workloads.custom("noalloc", 2, 8, 2, 1000, 128, True, "llm", 500, 0, seed=seed)
    q, k, v = workloads.generate(w)
    return tuple((t.float() * scale).to(torch.bfloat16).cuda() for t in (q, k, v))


def test_noalloc_quantize_matches_workspace_quantize_on_consecutive_calls():
    for scale, seed in ((40.0, 1), (0.03, 2)):       # second call: smaller amax, same scratch words
        q, k, v = _inputs(scale, seed)
        ref = mq.quantize(q, k, v)
        out = mq.alloc_quantized(mq.shape_of(q, k, True), q.device)
        for t in out.tensors.values():
            t.view(torch.uint8).fill_(0xA5)
        assert _quantize_noalloc(q, k, v, out) == 0
        status, word = mq.device_status()
        assert status == 0, hex(word)
        for f in mq.QUANT_FIELDS:
            a = ref[f].view(torch.uint8).cpu().numpy()
            b = out[f].view(torch.uint8).cpu().numpy()
            assert np.array_equal(a, b), f


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # B*Hq + B*Hkv + B*Hkv*d = 64*8 + 64*8 + 64*8*128 words > 65536
    q = torch.empty((64, 8, 128, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.empty((64, 8, 128, 128), dtype=torch.bfloat16, device="cuda")
    out = mq.alloc_quantized(mq.shape_of(q, k, True), q.device)
    assert _quantize_noalloc(q, k, k, out) == _lib.THRIFT_ERR_UNSUPPORTED
