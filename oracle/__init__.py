"""CPU oracle for the mixed FP4/BF16 attention forward.

TEST INFRASTRUCTURE: a plain, slow, FP64 (FP32 where a quantisation decision
is taken) numpy statement of what the library computes.  Only the tests, the
smoke check and the benchmark's CPU-baseline leg may import it; the CUDA
product path never does and shares no code with it.
"""
from . import attention, formats, quantize, select  # noqa: F401
