"""Oracle: the low-bit number formats (plain numpy, CPU).

TEST INFRASTRUCTURE.  Everything under ``oracle/`` is the slow, obviously
correct CPU statement of what the library computes.  Only the tests, the
smoke check and the benchmark's CPU-baseline leg may import it; the product
path never does.

Formats named on the pages: FP4 with block scales on Blackwell
(ThriftAttention: Selective Mixed Precision for Long-Context FP4 Attention,
abstract: "block-scaled quantisation techniques on Blackwell GPUs"; the
attention-quantization topic page lists NVFP4 and MXFP4 in its paper list
and FP8/FP4 in its overview).  The pages print no bit layouts, so the
standard definitions are written out here:

* e2m1 (FP4): sign, 2 exponent bits, 1 mantissa bit, bias 1, no inf/NaN.
  Magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}; code = 8*sign + index.
* e4m3 (OCP FP8 E4M3, "fn" variant): sign, 4 exponent bits (bias 7),
  3 mantissa bits, subnormals down to 2**-9, max 448, 0x7F/0xFF are NaN.

Rounding is round-to-nearest, ties to the even code, with saturation to the
largest finite value (no NaN is ever produced).  The sign of zero is kept.
"""
from __future__ import annotations

import numpy as np

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E4M3_MAX = 448.0


def e2m1_decode(codes) -> np.ndarray:
    """4-bit codes (0..15) -> float64 values."""
    c = np.asarray(codes).astype(np.int64)
    mag = E2M1_GRID[c & 7]
    return np.where((c & 8) != 0, -mag, mag)


def e2m1_encode(y) -> np.ndarray:
    """float -> 4-bit e2m1 code (uint8, 0..15), RNE with ties to even code, saturating.

    Between two neighbouring grid values the midpoint decides; a value exactly
    on a midpoint goes to the neighbour whose code is even (mantissa bit 0).
    """
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    # midpoints of the grid and whether the tie goes up (upper code even)
    code = np.zeros(a.shape, dtype=np.uint8)
    code = np.where(a > 0.25, 1, code)    # 0 | 0.5    tie -> 0 (code 0 even)
    code = np.where(a >= 0.75, 2, code)   # 0.5 | 1    tie -> 1 (code 2 even)
    code = np.where(a > 1.25, 3, code)    # 1 | 1.5    tie -> 1
    code = np.where(a >= 1.75, 4, code)   # 1.5 | 2    tie -> 2
    code = np.where(a > 2.5, 5, code)     # 2 | 3      tie -> 2
    code = np.where(a >= 3.5, 6, code)    # 3 | 4      tie -> 4
    code = np.where(a > 5.0, 7, code)     # 4 | 6      tie -> 4; above 6 saturates
    code = code.astype(np.uint8)
    return np.where(np.signbit(y), code | 8, code).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    """8-bit e4m3 codes -> float64 (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes).astype(np.int64)
    ef = (c >> 3) & 0xF
    man = c & 7
    sub = man.astype(np.float64) * 2.0 ** -9
    nrm = (1.0 + man / 8.0) * np.ldexp(1.0, ef - 7)
    mag = np.where(ef == 0, sub, nrm)
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return np.where((c & 0x80) != 0, -mag, mag)


def e4m3_encode(x) -> np.ndarray:
    """float -> e4m3 code (uint8), RNE ties-to-even, subnormals kept, saturating at 448.

    With E = max(floor(log2|x|), -6) the quantum is 2**(E-3); q = rint(|x| / quantum)
    is an exact scaling followed by numpy's round-half-even.  q == 16 carries into
    the next binade.  The code is then (E + 6) * 8 + q, which is also right for
    subnormals (E = -6, q < 8), clamped to 0x7E (448).
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e = np.frexp(a)                  # a = m * 2**e, m in [0.5, 1)
    E = np.where(a > 0, e - 1, -6)
    E = np.maximum(E, -6)
    q = np.rint(np.ldexp(a, 3 - E))     # exact scaling, RNE
    carry = q >= 16
    E = np.where(carry, E + 1, E)
    q = np.where(carry, q / 2, q)
    code = (E + 6) * 8 + q.astype(np.int64)
    code = np.minimum(code, 0x7E)
    code = np.where(np.signbit(x), code | 0x80, code)
    return code.astype(np.uint8)


def bf16_round(x) -> np.ndarray:
    """float64 -> nearest BF16 value (RNE), returned as float64."""
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)            # may double-round; only used for P emulation
    b = f.view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    b = (b + 0x7FFF + lsb) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32).astype(np.float64)
