"""Exact-arithmetic helpers for the tests (rational rounding to binary32)."""
from fractions import Fraction

import numpy as np


def round_f32(x: Fraction) -> np.float32:
    """The binary32 value nearest to the rational x, ties to even mantissa."""
    c = np.float32(float(x))
    best = None
    for cand in (np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))):
        if not np.isfinite(cand):
            continue
        d = abs(Fraction(float(cand)) - x)
        if best is None or d < best[0] or (d == best[0] and (int(np.float32(cand).view(np.uint32)) & 1) == 0):
            best = (d, cand)
    return np.float32(best[1])


def fma_f32(a, b, c) -> np.float32:
    """Single-rounding binary32 fused multiply-add."""
    return round_f32(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))
