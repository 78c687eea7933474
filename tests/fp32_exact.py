"""Exact IEEE-754 binary32 arithmetic on Python rationals.

Independent of the oracle and of the CUDA library: every operation is done
exactly on fractions.Fraction and rounded once to the nearest binary32 value
(ties to even).  Used to pin the oracle's fp32 routing arithmetic to its
definition (fused multiply-add chains, ascending-order sums).
"""
from fractions import Fraction

import numpy as np


def round_f32(x: Fraction) -> np.float32:
    if x == 0:
        return np.float32(0.0)
    sign = -1 if x < 0 else 1
    x = abs(x)
    e = x.numerator.bit_length() - x.denominator.bit_length()
    if Fraction(2) ** e > x:
        e -= 1
    e = max(e, -126)
    scaled = x / (Fraction(2) ** (e - 23))
    q = scaled.numerator // scaled.denominator
    rem = scaled - q
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and q % 2 == 1):
        q += 1
    return np.float32(sign * q * 2.0 ** (e - 23))


def F(v) -> Fraction:
    return Fraction(float(np.float32(v)))


def fma32(a, b, c) -> np.float32:
    return round_f32(F(a) * F(b) + F(c))


def add32(a, b) -> np.float32:
    return round_f32(F(a) + F(b))


def div32(a, b) -> np.float32:
    return round_f32(F(a) / F(b))


def dot_chain32(a, b) -> np.float32:
    acc = np.float32(0.0)
    for x, y in zip(a, b):
        acc = fma32(x, y, acc)
    return acc


def dot_tree32(a, b) -> np.float32:
    """Eight fma chains over the contiguous runs [l n / 8, (l + 1) n / 8) of the vectors, added as the balanced
    tree ((c0 + c1) + (c2 + c3)) + ((c4 + c5) + (c6 + c7)), every step rounded to fp32."""
    n = len(a)
    c = [dot_chain32(a[l * n // 8:(l + 1) * n // 8], b[l * n // 8:(l + 1) * n // 8]) for l in range(8)]
    return add32(add32(add32(c[0], c[1]), add32(c[2], c[3])), add32(add32(c[4], c[5]), add32(c[6], c[7])))
