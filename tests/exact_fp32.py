"""Exact rational arithmetic with explicit IEEE binary32 rounding.

Used by the oracle pins: each binary32 operation the quantization formulas
perform is evaluated exactly with ``fractions.Fraction`` and then rounded
once to the nearest binary32 value (ties to even), which is what IEEE-754
defines the hardware result to be. Nothing here calls the oracle or the CUDA
library, so it is an independent check of both.
"""

from __future__ import annotations

from fractions import Fraction

import numpy as np

_EMIN = -126  # smallest normal exponent of binary32
_P = 24       # binary32 precision (significand bits)


def rn32(q) -> Fraction:
    """Round an exact rational to the nearest binary32 value, ties to even."""
    q = Fraction(q)
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (max(e, _EMIN) - (_P - 1))
    n = round(a / ulp)  # Python rounds a Fraction half to even
    return sign * n * ulp


def f32(q: Fraction) -> np.float32:
    """A Fraction that is exactly a binary32 value, as np.float32 (checked)."""
    v = np.float32(float(q))
    assert Fraction(float(v)) == q, "value is not representable in binary32"
    return v


def rne_int(q: Fraction) -> int:
    """Round an exact rational to the nearest integer, ties to even."""
    return round(Fraction(q))


def exact_codes_row(v, mode: str, four_bit: bool):
    """The quantization formulas of one row, each binary32 operation rounded once.

    ``v``: sequence of binary32 inputs (already multiplied by smooth scales).
    Returns (codes list, scale Fraction, offset Fraction or None).
    """
    vals = [Fraction(float(np.float32(t))) for t in v]
    if mode == "symmetric":
        divisor = 7 if four_bit else 127
        lo, hi = (-7, 7) if four_bit else (-127, 127)
        amax = max(abs(t) for t in vals)
        scale = rn32(amax / divisor)
        if scale == 0:
            return [0] * len(vals), scale, None
        codes = [min(hi, max(lo, rne_int(rn32(t / scale)))) for t in vals]
        return codes, scale, None
    scale_opt, offset_opt = (15, 7) if four_bit else (255, 127)
    lo, hi = (-8, 7) if four_bit else (-128, 127)
    mx, mn = max(vals), min(vals)
    scale = rn32(rn32(mx - mn) / scale_opt)
    if scale == 0:
        return [offset_opt] * len(vals), scale, Fraction(offset_opt)
    offset = rn32(offset_opt - rn32(mx / scale))
    codes = [min(hi, max(lo, rne_int(rn32(rn32(t / scale) + offset)))) for t in vals]
    return codes, scale, offset
