"""libthrift: mixed FP4/BF16 attention forward (prefill) for NVIDIA B200 (sm_100a).

Most 128x128 query-key tile pairs run on block-scaled NVFP4 tensor cores,
a selected few (sink tile, diagonal tile, top-scoring pooled pairs) in
BF16, merged by one online softmax (ThriftAttention: Selective Mixed
Precision for Long-Context FP4 Attention, abstract; HyQuant:
Hybrid-Precision Quantization for LLM Attention, abstract).

The Python layer only marshals arguments into the C ABI of libthrift.so
(include/thrift.h); every step runs in the library's CUDA kernels.
"""
from ._lib import (FORMATS, OP_ATTN, OP_QUANTIZE, OP_QUANTIZE_MX, OP_SELECT, OP_SELECT_VERTICAL, QUANT_FIELDS, Quantized,  # noqa: F401
                   ThriftError, alloc_quantized, attention, attn_fwd, debug_withhold_v_load, decode_quantize_cache,
                   decode_step, device_status,
                   launch_count, lib, make_shape, probe_mma, quant_bytes, quantize, select, shape_of,
                   status_string, version, workspace_bytes)
from . import workloads  # noqa: F401
