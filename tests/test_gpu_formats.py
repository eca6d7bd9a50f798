"""GPU format probe: every finite BF16 bit pattern through the quantisation kernels,
against the oracle, bit for bit.

The 65,280 finite BF16 values (the 256 patterns with an all-ones exponent are left
out) fill one head of 510 rows x 128 channels twice: in ascending bit order, so that
each 16- or 32-element block holds neighbouring values of one binade, and in a seeded
random order, so that blocks mix magnitudes from the subnormals to 3.4e38.  The same
tensor serves as Q, K and V.  NVFP4 (`thrift_quantize`) and MXFP4
(`thrift_quantize_mx`) codes, scales and tensor scales, and V's FP8 codes, BF16 copy
and exponents must equal the oracle's (oracle/quantize.py, oracle/mx.py) -- the
rounding rules the library reads from the pages, including the sign kept on values
that round to zero and saturation at the largest code.
"""
import numpy as np
import pytest
import torch

import mixed_precision_bit_quant_b200 as mq
from test_gpu_mx import _check_quant as check_mx_quant
from test_gpu_parity import check_quantize

pytestmark = pytest.mark.gpu


def _all_finite_bf16() -> torch.Tensor:
    bits = np.arange(1 << 16, dtype=np.uint32)
    finite = ((bits >> 7) & 0xFF) != 0xFF
    vals = (bits[finite] << 16).view(np.float32)
    assert vals.size == 65280
    sorted_head = torch.from_numpy(vals.copy()).reshape(510, 128)
    perm = torch.randperm(vals.size, generator=torch.Generator().manual_seed(7))
    mixed_head = torch.from_numpy(vals.copy())[perm].reshape(510, 128)
    x = torch.stack([sorted_head, mixed_head]).unsqueeze(0)  # [1, 2, 510, 128]
    out = x.to(torch.bfloat16)
    # the cast is exact: every value is a BF16 value already
    assert torch.equal(out.float(), x)
    return out.contiguous()


def test_every_finite_bf16_nvfp4_and_fp8():
    x = _all_finite_bf16()
    xd = x.cuda()
    quant = mq.quantize(xd, xd, xd)
    st, word = mq.device_status()
    assert st == 0, f"device watchdog raised {word:#x}"
    check_quantize(x, x, x, quant.tensors)


def test_every_finite_bf16_mxfp4():
    x = _all_finite_bf16()
    xd = x.cuda()
    quant = mq.quantize(xd, xd, xd, fmt="mxfp4")
    st, word = mq.device_status()
    assert st == 0, f"device watchdog raised {word:#x}"
    check_mx_quant(x, x, x, quant)
