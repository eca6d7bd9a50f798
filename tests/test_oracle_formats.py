"""Pins for the oracle's e2m1 / e4m3 formats against independent definitions.

The e2m1 decode table is checked against the bit-field formula of the
format; e2m1 rounding against a brute-force nearest-value search; e4m3 against
torch's own float8_e4m3fn conversion (a library routine written elsewhere).
"""
import numpy as np
import pytest
import torch

from oracle.formats import (E2M1_GRID, bf16_round, e2m1_decode, e2m1_encode,
                            e4m3_decode, e4m3_encode)


def _e2m1_from_bits(code: int) -> float:
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1.0 + 0.5 * m)
    return -mag if s else mag


def test_e2m1_decode_matches_bitfield_formula():
    for c in range(16):
        got = float(e2m1_decode(np.array([c]))[0])
        want = _e2m1_from_bits(c)
        assert got == want and np.signbit(got) == np.signbit(want), c


def _nearest_e2m1(y: float) -> int:
    mags = [abs(_e2m1_from_bits(c)) for c in range(8)]
    a = min(abs(y), 6.0)
    best = min(range(8), key=lambda c: (abs(a - mags[c]), c & 1))
    return best | (8 if np.signbit(y) else 0)


def test_e2m1_encode_is_nearest_ties_even(rng):
    ys = list(rng.uniform(-8, 8, 4000))
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    ys += mids + [-m for m in mids] + list(E2M1_GRID) + [-g for g in E2M1_GRID] + [7.0, 100.0, -0.0, 1e-30]
    got = e2m1_encode(np.array(ys))
    want = np.array([_nearest_e2m1(y) for y in ys], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_e2m1_ties_listed():
    # tie cases: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    vals = e2m1_decode(e2m1_encode(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])))
    assert list(vals) == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]


def test_e2m1_roundtrip_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(e2m1_encode(e2m1_decode(codes)), codes)


def _torch_e4m3_codes(x: np.ndarray) -> np.ndarray:
    t = torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def test_e4m3_decode_matches_torch():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    ours = e4m3_decode(codes)
    theirs = torch.tensor(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, theirs)


def test_e4m3_encode_matches_torch_in_range(rng):
    reps = e4m3_decode(np.array([c for c in range(0x7F)], dtype=np.uint8))
    mids = (reps[1:] + reps[:-1]) / 2.0                      # every tie point
    xs = np.concatenate([
        rng.uniform(-448, 448, 20000),
        rng.uniform(-2.0 ** -6, 2.0 ** -6, 5000),            # subnormal range
        np.exp(rng.uniform(np.log(1e-4), np.log(448), 5000)),
        reps, -reps, mids, -mids,
    ]).astype(np.float32)
    assert np.array_equal(e4m3_encode(xs), _torch_e4m3_codes(xs))


def test_e4m3_saturates_and_roundtrips():
    big = np.array([448.0, 449.0, 464.0, 470.0, 1e6, -1e6])
    assert list(e4m3_decode(e4m3_encode(big))) == [448.0, 448.0, 448.0, 448.0, 448.0, -448.0]
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    back = e4m3_encode(e4m3_decode(codes))
    assert np.array_equal(back, codes)
    assert e4m3_decode(np.array([1]))[0] == 2.0 ** -9       # smallest subnormal


def test_bf16_round_matches_torch(rng):
    x = rng.standard_normal(5000) * np.exp(rng.uniform(-20, 20, 5000))
    ours = bf16_round(x)
    theirs = torch.tensor(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, theirs)
