"""Exact-arithmetic brute force for pinning the oracle.

Everything here works on Python Fractions, from the IEEE-754 definitions
(round to nearest, ties to even) rather than from any float routine, so that a
mistake in the oracle's C code (a dropped term, a reciprocal instead of a
division, a wrong rounding mode) cannot be reproduced here by accident.
"""
from fractions import Fraction

import numpy as np


def _f32_bits(v: np.float32) -> int:
    return int(np.array(v, np.float32).view(np.uint32))


def _nearest(target: Fraction, cands, even_key):
    best = None
    for c in cands:
        d = abs(Fraction(float(c)) - target)
        if best is None or d < best[0] or (d == best[0] and even_key(c) and not even_key(best[1])):
            best = (d, c)
    return best[1]


def fl32(x: Fraction) -> np.float32:
    """The fp32 value nearest to the exact rational x, ties to even."""
    c = np.float32(float(x))
    cands = {np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))}
    return _nearest(x, sorted(cands, key=float), lambda v: (_f32_bits(v) & 1) == 0)


def bf16(x: Fraction) -> int:
    """bf16 bit pattern nearest to the exact rational x, ties to even."""
    c = np.float32(float(x))
    hi = _f32_bits(c) >> 16
    cands = []
    for h in (hi - 1, hi, hi + 1, hi + 2):
        h &= 0xFFFF
        v = np.array(h << 16, np.uint32).view(np.float32)
        if np.isfinite(v):
            cands.append(h)
    best = None
    for h in cands:
        v = Fraction(float(np.array(h << 16, np.uint32).view(np.float32)))
        d = abs(v - x)
        if best is None or d < best[0] or (d == best[0] and (h & 1) == 0 and (best[1] & 1) == 1):
            best = (d, h)
    return best[1]


def bf16_value(h: int) -> Fraction:
    return Fraction(float(np.array(int(h) << 16, np.uint32).view(np.float32)))


def round_half_even(x: Fraction) -> int:
    f = x.numerator // x.denominator      # floor
    r = x - f
    if r > Fraction(1, 2):
        return f + 1
    if r < Fraction(1, 2):
        return f
    return f if f % 2 == 0 else f + 1


EPS = fl32(Fraction(1, 10**8))


def quantize_row_exact(vals):
    """vals: list of Fractions (exact bf16 or fp32 values) -> (q list, s float32)."""
    a = max(abs(v) for v in vals)
    clipped = a if a > Fraction(float(EPS)) else Fraction(float(EPS))
    s = fl32(clipped / 127)
    S = Fraction(float(s))
    q = []
    for v in vals:
        r = round_half_even(Fraction(float(fl32(v / S))))
        q.append(max(-127, min(127, r)))
    return q, s


def epilogue_exact(acc: int, s_row, s_col, bias_h=None) -> int:
    f = fl32(Fraction(acc))
    f = fl32(Fraction(float(f)) * Fraction(float(s_row)))
    f = fl32(Fraction(float(f)) * Fraction(float(s_col)))
    if bias_h is not None:
        f = fl32(Fraction(float(f)) + bf16_value(bias_h))
    return bf16(Fraction(float(f)))
