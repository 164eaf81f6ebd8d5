"""Exact rational arithmetic for pinning the oracle (test helper, not the oracle).

Everything here is computed with Python's Fraction, independently of the
oracle's binary32 arithmetic, and rounded to binary32 by its own
round-half-to-even routine.
"""
from fractions import Fraction
import math

import numpy as np


def F(v) -> Fraction:
    """Exact value of a binary32/binary64 number."""
    return Fraction(float(v))


def round_to_f32(fr: Fraction) -> np.float32:
    """The binary32 value nearest to fr, ties to even (normal and subnormal range)."""
    if fr == 0:
        return np.float32(0.0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    # now 2^e <= a < 2^(e+1)
    q = max(e, -126) - 23                      # exponent of the quantum
    n = a / (Fraction(2) ** q)
    fl = math.floor(n)
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    v = sign * fl * (Fraction(2) ** q)
    out = np.float32(float(v))
    assert F(out) == v, "value not representable: overflow"
    return out


def ulp32(v) -> float:
    v = abs(float(v))
    if v < 2.0 ** -126:
        return 2.0 ** -149
    return 2.0 ** (math.floor(math.log2(v)) - 23)


def round_half_even(fr: Fraction) -> int:
    fl = math.floor(fr)
    rem = fr - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        return fl + 1
    return fl


def exact_codes(x, lo, s):
    """q_k = clamp(round(exact (x_k - lo) / s), 0, 15) and the distance of each exact
    quotient to the nearest half-integer (to skip near-ties)."""
    if float(s) == 0.0:
        return [0] * len(x), [1.0] * len(x)
    qs, gaps = [], []
    for xk in x:
        y = (F(xk) - F(lo)) / F(s)
        q = min(max(round_half_even(y), 0), 15)
        frac = y - math.floor(y)
        gaps.append(abs(float(frac) - 0.5))
        qs.append(q)
    return qs, gaps


def exact_loss(x, lo, s, qs):
    """sum_k (x_k - (q_k*s + lo))^2 exactly, and the elementwise errors."""
    errs = [F(xk) - (q * F(s) + F(lo)) for xk, q in zip(x, qs)]
    return sum(e * e for e in errs), errs


def loss_error_bound(x, lo, s, qs, errs, d):
    """Bound on |binary32 pipeline - exact| for the loss: one rounding of the
    reconstruction, of the error, of its square, and log2(P) levels of the
    pairwise sum (first order, times a safety factor of 4)."""
    u = 2.0 ** -24
    p = 1
    while p < d:
        p *= 2
    levels = max(int(math.log2(p)), 0)
    tot = 0.0
    sq = 0.0
    for q, e in zip(qs, errs):
        xh = abs(q * float(s) + float(lo))
        ea = abs(float(e))
        tot += 2 * ea * (u * xh + u * (ea + u * xh)) + (u * xh) ** 2
        sq += ea * ea
    tot += (levels + 2) * u * sq
    return 4 * tot + 2.0 ** -149
