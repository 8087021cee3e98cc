"""Exact-arithmetic helpers for the oracle pins (rationals, correctly rounded
binary32).  Independent of the oracle's C code: these follow IEEE-754's
definition of round-to-nearest-even directly on fractions."""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def round_binary(fr: Fraction, mant: int, emin: int) -> Fraction:
    """Nearest (ties-to-even) value with `mant` fraction bits and minimum normal
    exponent `emin` (subnormals kept); no overflow handling."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    quantum = Fraction(2) ** (e - mant)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * quantum


def fp32(fr: Fraction) -> float:
    return float(round_binary(Fraction(fr), 23, -126))


def quantize_exact(x: float, amax: float) -> tuple[int, float]:
    """Per-block INT8 code of x in a block whose max |.| is amax, with every
    binary32 rounding of the quantiser done exactly on rationals:
    s = fp32(127/amax), y = fp32(x*s), code = clamp(rne(y), +-127),
    delta = fp32(amax/127)."""
    if amax == 0:
        return 0, 0.0
    s = fp32(Fraction(127) / Fraction(amax))
    y = fp32(Fraction(x) * Fraction(s))
    c = round(y)  # Python's round on a float is round-half-to-even
    c = max(-127, min(127, c))
    return int(c), fp32(Fraction(amax) / 127)


def all_finite_fp16() -> np.ndarray:
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16)
    return vals[np.isfinite(vals)]
