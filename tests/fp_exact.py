"""Exact-arithmetic helpers for pinning the oracle (no floating-point
arithmetic of the machine is trusted here).

``round_to_f32`` rounds an exact rational to the nearest IEEE-754 binary32
value, ties to even, with gradual underflow and overflow to infinity, using
only integer arithmetic.  ``round_to_bf16_bits`` does the same for bfloat16
(8 significant bits, binary32's exponent range).
"""
from fractions import Fraction

import numpy as np


def _round_rational(x: Fraction, mant_bits: int, emin: int, emax: int):
    """Return (sign, integer significand M, exponent E) with value M * 2**E,
    rounded to ``mant_bits`` significant bits (ties to even), or None for
    overflow.  emin: exponent of the smallest normal; subnormals share it."""
    if x == 0:
        return (0, 0, 0)
    sign = 1 if x < 0 else 0
    a = -x if sign else x
    # e with 2**e <= a < 2**(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, emin)                       # below the normal range: fixed quantum
    quantum_exp = e - (mant_bits - 1)
    scaled = a / (Fraction(2) ** quantum_exp)
    q, r = divmod(scaled.numerator, scaled.denominator)
    twice = 2 * r
    if twice > scaled.denominator or (twice == scaled.denominator and (q & 1)):
        q += 1
    if q == 1 << mant_bits:                # carried into the next binade
        q >>= 1
        quantum_exp += 1
    if quantum_exp + (mant_bits - 1) > emax:
        return None
    return (sign, q, quantum_exp)


def round_to_f32(x: Fraction) -> np.float32:
    r = _round_rational(Fraction(x), 24, -126, 127)
    if r is None:
        return np.float32(-np.inf if x < 0 else np.inf)
    sign, q, e = r
    val = float(Fraction(q) * (Fraction(2) ** e))   # exact in binary64
    return np.float32(-val if sign else val)


def f32_exact(x) -> Fraction:
    return Fraction(float(np.float32(x)))


def bf16_bits_to_fraction(bits: int) -> Fraction:
    return Fraction(float((np.uint32(bits) << np.uint32(16)).view(np.float32)))


def round_to_bf16_bits(x: Fraction) -> int:
    """Nearest bf16 (ties to even) of an exact rational, as a bit pattern."""
    r = _round_rational(Fraction(x), 8, -126, 127)
    neg = x < 0
    if r is None:
        return 0xFF80 if neg else 0x7F80
    sign, q, e = r
    val = np.float32(float(Fraction(q) * (Fraction(2) ** e)))
    bits = int(np.array([val], dtype=np.float32).view(np.uint32)[0]) >> 16
    if neg:
        bits |= 0x8000
    return bits
