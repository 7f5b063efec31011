"""Exact-arithmetic helpers used to pin the oracle.

These compute the defining real-number results with Python's ``Fraction``
(no floating point anywhere) and round them with an explicit
round-half-to-even rule, so they share nothing with the oracle's IEEE
binary32 arithmetic or its software binary16 conversion.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def half_value(bits: int) -> Fraction | None:
    """Exact value of a finite binary16 bit pattern (None for Inf / NaN)."""
    sign = -1 if bits & 0x8000 else 1
    e = (bits >> 10) & 0x1F
    f = bits & 0x3FF
    if e == 31:
        return None
    if e == 0:
        return sign * Fraction(f, 1 << 24)
    return sign * Fraction(1024 + f) * Fraction(2) ** (e - 25)


def round_half_even(q: Fraction) -> int:
    n = q.numerator // q.denominator  # floor
    r = q - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return n


def _binade(a: Fraction) -> int:
    """E with 2**E <= a < 2**(E+1), for a > 0."""
    E = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** E > a:
        E -= 1
    while Fraction(2) ** (E + 1) <= a:
        E += 1
    return E


def round_to_half_bits(q: Fraction) -> int:
    """Nearest binary16 to the exact value q, ties to even, overflow to Inf."""
    sign = 0x8000 if q < 0 else 0
    a = -q if q < 0 else q
    if a == 0:
        return sign
    E = _binade(a)
    if E < -14:
        n = round_half_even(a * (1 << 24))  # multiple of 2^-24
        return sign | n                       # n == 1024 is the smallest normal
    n = round_half_even(a / Fraction(2) ** (E - 10))  # in [1024, 2048]
    if n == 2048:
        n, E = 1024, E + 1
    if E > 15:
        return sign | 0x7C00
    return sign | ((E + 15) << 10) | (n - 1024)


def e5m2_table():
    """(byte, exact value) for every finite E5M2 code, from the format definition:
    sign, 5-bit exponent with bias 15, 2-bit fraction, subnormal step 2^-16."""
    out = []
    for b in range(256):
        e = (b >> 2) & 0x1F
        f = b & 3
        if e == 31:
            continue
        mag = Fraction(f, 1 << 16) if e == 0 else Fraction(4 + f, 4) * Fraction(2) ** (e - 15)
        out.append((b, -mag if b & 0x80 else mag))
    return out


def e5m2_nearest_all(bits: np.ndarray) -> np.ndarray:
    """Brute force over every finite E5M2 magnitude: the byte nearest to each
    binary16 input, ties to the even fraction.  Magnitudes at or beyond the
    midpoint between 57344 and the next step 65536 (fraction 00, even) go to
    Inf.  NaN -> sign | 0x7E, Inf -> sign | 0x7C.  All values and differences
    are dyadic rationals with < 53 significant bits, so float64 is exact here."""
    bits = np.asarray(bits, dtype=np.uint16)
    mags = [(b, float(v)) for b, v in e5m2_table() if not b & 0x80]
    cand_b = np.array([b for b, _ in mags] + [0x7C], dtype=np.int64)
    cand_v = np.array([v for _, v in mags] + [65536.0])
    vals = np.abs(bits.view(np.float16).astype(np.float64))
    with np.errstate(invalid="ignore"):
        d = np.abs(vals[:, None] - cand_v[None, :])
    dmin = d.min(axis=1, keepdims=True)
    tie_ok = (d == dmin) & ((cand_b[None, :] & 1) == 0)
    has_even = tie_ok.any(axis=1)
    pick = np.where(has_even, np.argmax(tie_ok, axis=1), np.argmin(d, axis=1))
    out = cand_b[pick]
    sign = np.where(bits & 0x8000, 0x80, 0)
    e = (bits >> 10) & 0x1F
    nan = (e == 31) & ((bits & 0x3FF) != 0)
    inf = (e == 31) & ((bits & 0x3FF) == 0)
    out = np.where(nan, 0x7E, np.where(inf, 0x7C, out))
    return (out | sign).astype(np.uint8)


def half_bits(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float16).view(np.uint16)
