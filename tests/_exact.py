"""Exact rational helpers for the oracle pins (independent of the oracle's C).

Everything here is written from the IEEE-754 definitions with Python's
``fractions.Fraction``; none of it is shared with the oracle or the CUDA path.
"""
from fractions import Fraction

import numpy as np

F32_MAX = Fraction(2) ** 127 * (2 - Fraction(1, 2 ** 23))


def frac_f32(x) -> Fraction:
    return Fraction(float(np.float32(x)))


def f32_rn(x: Fraction) -> np.float32:
    """Round an exact rational to the nearest fp32, ties to even."""
    if x == 0:
        return np.float32(0.0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    # overflow: beyond the midpoint between F32_MAX and 2^128
    if a >= Fraction(2) ** 128 - Fraction(2) ** 103:
        return np.float32(sign * np.inf)
    c = np.float32(float(a))  # within an ulp or two of the answer
    cands = {c}
    for _ in range(2):
        for v in list(cands):
            cands.add(np.nextafter(v, np.float32(np.inf)))
            cands.add(np.nextafter(v, np.float32(0)))
    best = None
    for v in sorted(cands, key=float):
        if not np.isfinite(v):
            continue
        d = abs(Fraction(float(v)) - a)
        if best is None or d < best[0] or (
                d == best[0] and (np.float32(v).view(np.uint32) & 1) == 0):
            best = (d, v)
    return np.float32(sign * best[1])


def argmin_nearest(T, u) -> int:
    """Lowest index j minimising |u - T_j| exactly."""
    uf = frac_f32(u)
    best, bd = 0, None
    for j, t in enumerate(T):
        d = abs(uf - frac_f32(t))
        if bd is None or d < bd:
            best, bd = j, d
    return best


def total_order_keys(u_f32: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(u_f32, dtype=np.float32).view(np.uint32)
    neg = (b >> np.uint32(31)).astype(bool)
    return np.where(neg, ~b, b | np.uint32(0x80000000)).astype(np.uint32)
