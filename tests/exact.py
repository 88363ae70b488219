"""Exact rational arithmetic for pinning the oracle (tests only).

Rounding to a binary floating-point format is written here from the IEEE 754
definition on ``fractions.Fraction`` values, independently of the C oracle:
the result is the representable number nearest to x, ties to the one with an
even integral significand; magnitudes at or beyond the overflow threshold give
infinity.
"""
from __future__ import annotations

import math
import struct
from fractions import Fraction

INF = float("inf")


def _floor_log2(a: Fraction) -> int:
    e = a.numerator.bit_length() - a.denominator.bit_length()
    # adjust so that 2^e <= a < 2^(e+1)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    return e


def round_binary(x: Fraction, prec: int, emin: int, emax: int):
    """Round x to a binary format with ``prec`` significand bits (implicit bit
    included), minimum normal exponent ``emin`` and maximum exponent ``emax``.
    Returns a Fraction, or +-INF on overflow."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = max(_floor_log2(a), emin)
    quantum = Fraction(2) ** (e - prec + 1)
    n = a / quantum
    fl = math.floor(n)
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    r = fl * quantum
    max_finite = (2 - Fraction(2) ** (1 - prec)) * Fraction(2) ** emax
    if r > max_finite:
        return sign * INF
    return sign * r


def rn32(x: Fraction):
    return round_binary(x, 24, -126, 127)


def rn16(x: Fraction):
    return round_binary(x, 11, -14, 15)


def rnbf16(x: Fraction):
    return round_binary(x, 8, -126, 127)


def f32_bits(v: float) -> int:
    return struct.unpack("<I", struct.pack("<f", v))[0]


def nearest_int_even(t: Fraction, lo: int, hi: int) -> int:
    """Integer in [lo, hi] nearest to t; of two equally near, the even one.
    Found by enumerating every candidate."""
    best = None
    for q in range(lo, hi + 1):
        d = abs(t - q)
        if best is None or d < best[0] or (d == best[0] and q % 2 == 0):
            best = (d, q)
    return best[1]


def kth_smallest_by_counting(vals, k: int):
    """The unique v among vals with #{x < v} < k <= #{x <= v} (no sorting)."""
    for v in vals:
        below = sum(1 for x in vals if x < v)
        at_or_below = sum(1 for x in vals if x <= v)
        if below < k <= at_or_below:
            return v
    raise AssertionError("no order statistic found")


def quantize_group_exact(ws, qbits: int, p_k: int, export: bool):
    """Reference for one group from exact arithmetic.

    ``ws`` are the group's binary32 values (Python floats), ``p_k`` the rank k.
    Returns dict(clip, s, h, q, dq) as Fractions (h: the binary16 scale value,
    or None in training mode); raises OverflowError on a binary16 overflow.
    """
    qmax = 31 if qbits == 6 else 127
    F = [Fraction(w) for w in ws]
    c = kth_smallest_by_counting([abs(x) for x in F], p_k)
    s32 = rn32(c / qmax)
    h = None
    s = s32
    if export:
        h = rn16(s32)
        if h in (INF, -INF):
            raise OverflowError("binary16 scale overflow")
        s = h
    qs, dqs = [], []
    for x in F:
        if s == 0:
            q = 0
        else:
            wc = min(max(x, -c), c)
            t = rn32(wc / s)
            q = nearest_int_even(t, -qmax, qmax) if abs(t) <= qmax + 1 else (qmax if t > 0 else -qmax)
        qs.append(q)
        dqs.append(rn32(q * s))
    return dict(clip=c, s=s, h=h, q=qs, dq=dqs)
