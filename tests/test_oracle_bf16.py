"""Pins for the oracle's fp32 -> bf16 conversion (round to nearest, ties to even).

The step writes its updated fp32 master weights as bf16 into the buffer that
the parameter all-gather fills ("CS336 lecture 8", ZeRO-1 code sketch, the
final all-gather; 2-byte bf16 parameters in the 16 bytes/param ledger).  The
rounding rule itself is IEEE-754's default, applied to bfloat16.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from fp_exact import bf16_bits_to_fraction, round_to_bf16_bits


def bits_f32(u: int) -> np.float32:
    return np.array([u], dtype=np.uint32).view(np.float32)[0]


@pytest.mark.parametrize("f32_bits, bf16_bits", [
    (0x3F800000, 0x3F80),   # 1.0
    (0x3F808000, 0x3F80),   # tie between 0x3F80 and 0x3F81 -> even 0x3F80
    (0x3F818000, 0x3F82),   # tie between 0x3F81 and 0x3F82 -> even 0x3F82
    (0x3F808001, 0x3F81),   # just above the tie -> up
    (0x3F807FFF, 0x3F80),   # just below the tie -> down
    (0xBF818000, 0xBF82),   # negative tie -> even (magnitude up)
    (0x00000000, 0x0000),   # +0
    (0x80000000, 0x8000),   # -0 keeps its sign
    (0x00000001, 0x0000),   # smallest fp32 subnormal rounds to +0
    (0x00010000, 0x0001),   # smallest bf16 subnormal is exact
    (0x00018000, 0x0002),   # subnormal tie -> even
    (0x7F800000, 0x7F80),   # +inf
    (0xFF800000, 0xFF80),   # -inf
    (0x7F7FFFFF, 0x7F80),   # largest fp32 finite overflows bf16 -> +inf
    (0x7F7F7FFF, 0x7F7F),   # below the overflow threshold stays finite
    (0x7F7F8000, 0x7F80),   # tie at the top rounds to even = +inf
])
def test_hand_picked(f32_bits, bf16_bits):
    assert oracle.f32_to_bf16(bits_f32(f32_bits)) == bf16_bits


@pytest.mark.parametrize("nan_bits", [0x7FC00000, 0x7F800001, 0xFFC12345, 0x7FFFFFFF])
def test_nan_stays_nan_and_quiet(nan_bits):
    h = oracle.f32_to_bf16(bits_f32(nan_bits))
    assert (h & 0x7F80) == 0x7F80 and (h & 0x007F) != 0, hex(h)
    assert (h & 0x0040) != 0                     # quiet
    assert (h >> 15) == (nan_bits >> 31)         # sign kept


def test_widening_is_exact():
    for h in [0x0000, 0x8000, 0x0001, 0x3F80, 0x7F7F, 0xC2F7, 0x7F80, 0xFF80]:
        assert np.float32(oracle.bf16_to_f32(h)).view(np.uint32) == (h << 16)


def test_against_exact_rational_rounding():
    """Random fp32 patterns (all binades, both signs): the oracle equals the
    nearest-even bf16 computed in exact rational arithmetic."""
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 1 << 32, size=4000, dtype=np.uint64).astype(np.uint32)
    # include the neighbourhoods of ties
    ties = (rng.integers(0, 1 << 16, size=1000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    bits = np.concatenate([bits, ties, ties + 1, ties - 1])
    vals = bits.view(np.float32)
    ours = oracle.f32_to_bf16_array(vals)
    for v, h in zip(vals, ours):
        if not np.isfinite(v):
            continue
        want = round_to_bf16_bits(Fraction(float(v)))
        if float(v) == 0.0:
            want = 0x8000 if np.signbit(v) else 0
        elif Fraction(float(v)) != 0 and want in (0, 0x8000) and np.signbit(v):
            want = 0x8000
        assert int(h) == want, (hex(int(np.array([v]).view(np.uint32)[0])), hex(int(h)), hex(want))


def test_against_torch_on_finite_values():
    """Library special case: torch's CPU bfloat16 conversion is also RNE."""
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 1 << 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    vals = bits.view(np.float32)
    vals = vals[np.isfinite(vals)]
    ours = oracle.f32_to_bf16_array(vals)
    theirs = torch.from_numpy(vals.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)


def test_round_trip_of_bf16_values_is_identity():
    h = np.arange(0, 1 << 16, dtype=np.uint32)
    h = h[((h & 0x7F80) != 0x7F80) | ((h & 0x7F) == 0)]   # no NaNs
    back = oracle.f32_to_bf16_array(oracle.bf16_bits_to_f32(h.astype(np.uint16)))
    assert np.array_equal(back, h.astype(np.uint16))
    assert bf16_bits_to_fraction(0x3F80) == 1
