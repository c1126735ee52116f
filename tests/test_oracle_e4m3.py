"""Pins for the oracle's e4m3 decode and fp32 -> e4m3 encoder.

The oracle is pinned against things other than itself:
  * hand-worked landmark codes (tests/golden/e4m3_landmarks.json);
  * torch's own float8_e4m3fn conversions (an independent implementation of
    the same format), after clamping to +-448 so that torch's non-saturating
    cast and the saturating contract coincide;
  * closed-form properties (monotonicity, symmetry, exact round trip of all
    254 finite codes, ties to even at every midpoint).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle


def _finite_codes():
    return [c for c in range(256) if c not in (0x7F, 0xFF)]


def test_landmarks(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "e4m3_landmarks.json")))
    for code_s, val_s in fx["codes"].items():
        v = oracle.e4m3_decode(int(code_s, 16))
        if val_s == "nan":
            assert math.isnan(v)
        else:
            want = float(val_s)
            assert v == want, (code_s, v, want)
            if val_s.startswith("-"):
                assert math.copysign(1.0, v) < 0


def test_decode_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if math.isnan(ref[c]):
            assert math.isnan(v), c
        else:
            assert v == ref[c], (c, v, ref[c])
            assert math.copysign(1.0, v) == math.copysign(1.0, ref[c]), c


def test_decode_closed_form_properties():
    pos = [oracle.e4m3_decode(c) for c in range(0x00, 0x7F)]
    # strictly increasing over the positive codes, from 0 to 448
    assert all(b > a for a, b in zip(pos, pos[1:]))
    assert pos[0] == 0.0 and pos[-1] == 448.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9       # smallest subnormal
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6       # smallest normal
    for c in range(0x7F):
        assert oracle.e4m3_decode(c | 0x80) == -oracle.e4m3_decode(c)
    # every finite value times 2^9 is an integer (the oracle's int64 GEMM relies on it)
    for c in _finite_codes():
        v = oracle.e4m3_decode(c) * 512
        assert v == int(v)


def test_encode_roundtrip_all_finite_codes():
    for c in _finite_codes():
        v = oracle.e4m3_decode(c)
        got = oracle.e4m3_encode(v)
        if v == 0.0:
            assert got == c  # +0 -> 0x00, -0 -> 0x80
        else:
            assert got == c, (hex(c), v, hex(got))


def test_encode_midpoints_ties_to_even():
    # between each pair of adjacent positive values the midpoint goes to the
    # code with an even mantissa; just above/below go to the nearer one.
    pos = [oracle.e4m3_decode(c) for c in range(0x00, 0x7F)]
    for c in range(len(pos) - 1):
        lo, hi = pos[c], pos[c + 1]
        mid = (lo + hi) / 2  # exact in fp32: both are short binary fractions
        assert np.float32(mid) == mid
        even = c if (c & 1) == 0 else c + 1
        assert oracle.e4m3_encode(mid) == even, (lo, hi)
        assert oracle.e4m3_encode(-mid) == (even | 0x80)
        below = float(np.nextafter(np.float32(mid), np.float32(0)))
        above = float(np.nextafter(np.float32(mid), np.float32(1e9)))
        assert oracle.e4m3_encode(below) == c
        assert oracle.e4m3_encode(above) == c + 1


def test_encode_saturation_and_specials():
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(463.99) == 0x7E
    assert oracle.e4m3_encode(464.0) == 0x7E        # tie 448/480 -> even -> 448
    assert oracle.e4m3_encode(465.0) == 0x7E        # would be 480: saturates
    assert oracle.e4m3_encode(1e30) == 0x7E
    assert oracle.e4m3_encode(float("inf")) == 0x7E
    assert oracle.e4m3_encode(-float("inf")) == 0xFE
    assert oracle.e4m3_encode(-1e30) == 0xFE
    assert oracle.e4m3_encode(0.0) == 0x00
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(1e-30) == 0x00
    assert oracle.e4m3_encode(-1e-30) == 0x80
    assert oracle.e4m3_encode(float("nan")) == 0x7F


def _torch_encode_bits(bits: np.ndarray) -> np.ndarray:
    f = torch.from_numpy(bits.view(np.int32)).view(torch.float32)
    return f.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _compare_range(bits: np.ndarray):
    bits = np.ascontiguousarray(bits, dtype=np.uint32)
    f = bits.view(np.float32)
    keep = ~np.isnan(f)                       # NaN inputs are outside the contract
    got = oracle.e4m3_encode_bits(bits)
    want = _torch_encode_bits(bits)
    bad = np.nonzero((got != want) & keep)[0]
    assert bad.size == 0, [(hex(int(bits[i])), float(f[i]), hex(int(got[i])), hex(int(want[i])))
                           for i in bad[:8]]


def test_encode_exhaustive_rounding_range():
    """Every fp32 pattern whose magnitude lies in [2^-27, 2^10): all values
    that do not trivially flush to zero or saturate, both signs."""
    for biased_exp in range(100, 137):
        base = np.uint32(biased_exp << 23)
        mant = np.arange(1 << 23, dtype=np.uint32)
        pos = base | mant
        _compare_range(pos)
        _compare_range(pos | np.uint32(0x80000000))


def test_encode_strided_full_range():
    """A stride-4093 sample over all 2^32 patterns (covers fp32 subnormals,
    huge values, infinities)."""
    bits = np.arange(0, 1 << 32, 4093, dtype=np.uint64).astype(np.uint32)
    _compare_range(bits)
    _compare_range(np.array([0x7F800000, 0xFF800000, 0x00000001, 0x80000001,
                             0x007FFFFF, 0x00800000, 0x3A800000, 0x3A800001,
                             0x3A7FFFFF], dtype=np.uint32))
