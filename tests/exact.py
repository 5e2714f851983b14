"""Exact-arithmetic helpers for the oracle pins (independent of the oracle).

Rounding a rational number to the nearest fp32 / bf16 value is done here by
exact comparison of Fractions, so the pins do not inherit any rounding of the
code under test.
"""
from fractions import Fraction

import numpy as np


def _neighbours_f32(x: float):
    f = np.float32(x)
    lo = np.nextafter(f, np.float32(-np.inf), dtype=np.float32)
    hi = np.nextafter(f, np.float32(np.inf), dtype=np.float32)
    return [lo, f, hi]


def nearest_f32(q: Fraction) -> np.float32:
    """Round an exact rational to the nearest fp32, ties to even mantissa."""
    if q == 0:
        return np.float32(0.0)
    best = None
    for c in _neighbours_f32(float(q)):
        if not np.isfinite(c):
            continue
        d = abs(Fraction(float(c)) - q)
        if best is None or d < best[0]:
            best = (d, c)
        elif d == best[0]:
            # tie: pick the even mantissa
            if int(np.float32(c).view(np.uint32)) % 2 == 0:
                best = (d, c)
    return np.float32(best[1])


def rint_half_even(q: Fraction) -> int:
    """Round an exact rational to the nearest integer, ties to even."""
    fl = q.numerator // q.denominator
    rem = q - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def f32_div(a, b) -> np.float32:
    """IEEE fp32 division a / b (exactly rounded), for fp32 inputs."""
    return nearest_f32(Fraction(float(a)) / Fraction(float(b)))


def f32_mul(a, b) -> np.float32:
    return nearest_f32(Fraction(float(a)) * Fraction(float(b)))
