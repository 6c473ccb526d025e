"""Exact-arithmetic helpers for the oracle pins (independent of the oracle).

Values are decoded here from the OCP bit fields (not from a table) and rounded
with rational arithmetic, so a mistake in the oracle's tables, its rounding or
its operation order shows up as a mismatch.
"""
import math
from fractions import Fraction

import numpy as np


def e2m1_from_bits(code: int) -> Fraction:
    """OCP E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0."""
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        v = Fraction(m, 2)                    # subnormal: 0.m * 2^(1-1)
    else:
        v = Fraction(2) ** (e - 1) * (1 + Fraction(m, 2))
    return -v if s else v


def e4m3_from_bits(byte: int):
    """OCP E4M3FN: sign, 4 exponent bits (bias 7), 3 mantissa bits; S.1111.111 NaN."""
    s = (byte >> 7) & 1
    e = (byte >> 3) & 15
    m = byte & 7
    if e == 15 and m == 7:
        return None
    if e == 0:
        v = Fraction(m, 8) * Fraction(2) ** -6
    else:
        v = (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
    return -v if s else v


def pow2(e: int) -> Fraction:
    return Fraction(2) ** e


def rn32(x: Fraction) -> np.float32:
    """Correctly rounded (nearest, ties to even) fp32 of an exact rational."""
    if x == 0:
        return np.float32(0.0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while pow2(e) > a:
        e -= 1
    while pow2(e + 1) <= a:
        e += 1
    q = max(e, -126) - 23                    # weight of the last kept bit
    m = a / pow2(q)
    n = m.numerator // m.denominator
    r = m - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    val = n * pow2(q)
    if val >= pow2(128):
        return np.float32(sign * np.inf)
    return np.float32(sign * float(val))


def frac32(x) -> Fraction:
    return Fraction(float(np.float32(x)))


def row_values(codes_row: np.ndarray, scales_row: np.ndarray):
    """Exact dequantised values of one MXFP4 row (codes n/2 bytes, scales n/32)."""
    n = codes_row.shape[0] * 2
    out = []
    for e in range(n):
        b = int(codes_row[e // 2])
        c = (b >> 4) if (e & 1) else (b & 15)
        out.append(e2m1_from_bits(c) * pow2(int(scales_row[e // 32]) - 127))
    return out


def exact_score(kc, ks, qc, qs, w) -> np.float32:
    """Indexer score from exact rationals: d_h rounded once, fp32 fma chain."""
    k = row_values(kc, ks)
    d = []
    for h in range(4):
        q = row_values(qc[h], qs[h])
        d.append(rn32(sum(qi * ki for qi, ki in zip(q, k))))
    s = rn32(frac32(w[0]) * frac32(d[0]))
    for h in range(1, 4):
        s = rn32(frac32(w[h]) * frac32(d[h]) + frac32(s))
    if s == 0:
        s = np.float32(0.0)
    return s


def brute_block(x):
    """Independent MXFP4 block encoder: exhaustive scale search + nearest code."""
    x = np.asarray(x, np.float32)
    amax = float(np.max(np.abs(x)))
    if amax == 0.0:
        X = -127
    else:
        X = None
        for cand in range(-200, 200):
            if 4.0 <= amax * 2.0 ** (-cand) < 8.0:
                X = cand
                break
        X = max(-127, min(127, X))
    grid = [float(e2m1_from_bits(c)) for c in range(8)]
    codes = []
    for v in x:
        a = abs(float(v)) * 2.0 ** (-X)
        best = None
        for i, g in enumerate(grid):
            d = abs(a - g)
            if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
                best = (d, i)
        i = 7 if a >= 6.0 else best[1]
        codes.append(i | (8 if math.copysign(1.0, float(v)) < 0 else 0))
    return codes, X + 127
