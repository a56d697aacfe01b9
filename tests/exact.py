"""Exact rational arithmetic with explicitly written IEEE rounding.

Used by the oracle pins to recompute, on tiny inputs, what the oracle computes
with numpy -- here from the definition of round-to-nearest-even on exact
rationals, so that the pins do not rest on numpy's floating point.
"""
from fractions import Fraction
import math


def rne_int(x: Fraction) -> int:
    """Round a rational to the nearest integer, ties to even."""
    f = math.floor(x)
    d = x - f
    if d > Fraction(1, 2):
        return f + 1
    if d < Fraction(1, 2):
        return f
    return f if f % 2 == 0 else f + 1


def _round_binary(x: Fraction, sig_bits: int, min_exp: int, max_exp: int) -> Fraction:
    """Round to a binary format with ``sig_bits`` significant bits (implicit bit
    included), smallest normal exponent ``min_exp`` and largest ``max_exp``.
    Returns a Fraction, or +-inf as a float when the result overflows."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = -x if x < 0 else x
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    # fix e so that 2^e <= a < 2^(e+1) exactly
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, min_exp)
    quantum = Fraction(2) ** (e - (sig_bits - 1))
    n = rne_int(a / quantum)
    r = n * quantum
    if r >= Fraction(2) ** (max_exp + 1):
        return sign * math.inf
    return sign * r


def to_f32(x: Fraction) -> Fraction:
    """IEEE binary32 round-to-nearest-even of an exact rational."""
    return _round_binary(Fraction(x), 24, -126, 127)


def to_bf16(x: Fraction) -> Fraction:
    """bfloat16 round-to-nearest-even of an exact rational."""
    return _round_binary(Fraction(x), 8, -126, 127)


def bf16_bits_of(x: Fraction) -> int:
    """bf16 bit pattern of an exactly representable bf16 value."""
    import numpy as np
    f = np.float32(float(x))
    assert Fraction(float(f)) == Fraction(x)
    return int(f.view(np.uint32)) >> 16
