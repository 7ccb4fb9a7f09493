"""Exact-rational model of IEEE-754 binary32 arithmetic (round to nearest, ties to even).

Used by the CPU tests to pin the oracle's fixed fp32 variation recipe: every
operation is evaluated exactly with fractions.Fraction and rounded once, which is
what IEEE fmaf / subtraction / sqrtf / scaling promise. Independent of both the
oracle and the GPU library.
"""
from fractions import Fraction
import math

import numpy as np

EMIN = -126          # smallest normal exponent
MANT = 23            # stored mantissa bits
MAX_F32 = (2 - Fraction(1, 2 ** MANT)) * Fraction(2) ** 127


def _floor_log2(x: Fraction) -> int:
    n, d = x.numerator, x.denominator
    e = n.bit_length() - d.bit_length()
    # adjust so that 2^e <= x < 2^(e+1)
    if Fraction(2) ** e > x:
        e -= 1
    elif Fraction(2) ** (e + 1) <= x:
        e += 1
    return e


def round_f32(x: Fraction) -> float:
    """Nearest binary32 to the exact rational x (ties to even), as a Python float."""
    if x == 0:
        return 0.0
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = max(_floor_log2(a), EMIN)
    quantum = Fraction(2) ** (e - MANT)
    q = a / quantum
    m = q.numerator // q.denominator
    rem = q - m
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and m % 2 == 1):
        m += 1
    r = m * quantum
    if r > MAX_F32:
        return sign * math.inf
    return sign * float(r)


def f(x) -> Fraction:
    return Fraction(float(np.float32(x)))


def fma(a, b, c) -> float:
    return round_f32(f(a) * f(b) + f(c))


def sub(a, b) -> float:
    return round_f32(f(a) - f(b))


def sqrt(a) -> float:
    """Correctly rounded binary32 square root of a non-negative binary32 value."""
    s = f(a)
    if s == 0:
        return 0.0
    r = float(np.float32(math.sqrt(float(s))))
    # walk to the binary32 value whose rounding interval contains sqrt(s)
    for _ in range(4):
        lo = float(np.nextafter(np.float32(r), np.float32(0)))
        hi = float(np.nextafter(np.float32(r), np.float32(np.inf)))
        mid_lo = (Fraction(lo) + Fraction(r)) / 2
        mid_hi = (Fraction(r) + Fraction(hi)) / 2
        if mid_lo * mid_lo > s:
            r = lo
        elif mid_hi * mid_hi < s:
            r = hi
        else:
            if mid_hi * mid_hi == s and (np.float32(r).view(np.uint32) & 1):
                r = hi
            elif mid_lo * mid_lo == s and (np.float32(r).view(np.uint32) & 1):
                r = lo
            return r
    raise AssertionError("sqrt did not converge")


def rne_int(x: Fraction) -> int:
    """Round an exact rational to the nearest integer, ties to even."""
    m = x.numerator // x.denominator
    rem = x - m
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and m % 2 == 1):
        m += 1
    return int(m)


def feature(P, k, v):
    """z = P [k; v]: per row an fp32 accumulator from 0 taking fma(P[i][j], x_j, acc), j ascending."""
    x = list(np.asarray(k, np.float32)) + list(np.asarray(v, np.float32))
    z = []
    for i in range(P.shape[0]):
        acc = 0.0
        for j, xj in enumerate(x):
            acc = fma(P[i, j], xj, acc)
        z.append(acc)
    return np.array(z, np.float32)


def quantised_step(zp, zc) -> int:
    s = 0.0
    for a, b in zip(zp, zc):
        di = sub(b, a)
        s = fma(di, di, s)
    r = sqrt(s)
    return rne_int(Fraction(r) * 2 ** 20)
