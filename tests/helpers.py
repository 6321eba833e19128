"""Exact-arithmetic helpers used by the tests to pin the CPU reference.

Nothing here is used by the product or by the reference itself.
"""
from __future__ import annotations

import math
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np


def f32_bits(v) -> int:
    return int(np.array(v, dtype=np.float32).view(np.uint32))


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    return (np.asarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _round_fraction(q: Fraction, mant_bits: int) -> Fraction:
    """Round a rational to the nearest binary float with `mant_bits` significant
    bits (ties to even), unbounded exponent (no overflow/underflow in use)."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    # fix e so that 2^e <= a < 2^(e+1)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - (mant_bits - 1))
    m = a / ulp
    lo = math.floor(m)
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sign * lo * ulp


def fraction_to_f32(q: Fraction) -> np.float32:
    """Correctly rounded fp32 of an exact rational."""
    r = _round_fraction(q, 24)
    return np.float32(float(r))  # r is exactly representable in fp32


def fraction_to_bf16_bits(q: Fraction) -> int:
    """Correctly rounded bf16 (bit pattern) of an exact rational."""
    r = _round_fraction(q, 8)
    return int(np.array(float(r), dtype=np.float32).view(np.uint32)) >> 16


def near_midpoint(q: Fraction, mant_bits: int, rel: float = 1e-9) -> bool:
    """True when q lies within rel of a rounding midpoint at mant_bits bits."""
    if q == 0:
        return False
    a = abs(q)
    r = _round_fraction(a, mant_bits)
    e = math.floor(math.log2(float(r))) if r else 0
    ulp = Fraction(2) ** (e - (mant_bits - 1))
    for mid in (r - ulp / 2, r + ulp / 2):
        if abs(a - mid) <= a * Fraction(rel):
            return True
    return False


def decimal_sigmoid(x: float, prec: int = 60) -> Fraction:
    """Logistic function evaluated with `prec` decimal digits (no libm)."""
    getcontext().prec = prec
    d = Decimal(x)
    v = Decimal(1) / (Decimal(1) + (-d).exp())
    return Fraction(v)


def decimal_tanh(x: Fraction, prec: int = 60) -> Fraction:
    getcontext().prec = prec
    d = Decimal(x.numerator) / Decimal(x.denominator)
    e2 = (2 * d).exp()
    return Fraction((e2 - 1) / (e2 + 1))


def exact_f32_dot(xb: np.ndarray, w: np.ndarray) -> Fraction:
    """Exact sum of bf16(x) * fp32(w) products as a rational."""
    xv = bf16_to_f32(xb).astype(np.float64)
    return sum((Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xv, w.astype(np.float64))),
               Fraction(0))
