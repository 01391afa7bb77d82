"""Exact binary32 rounding for CPU emulations of the kernels' fp32
sequences: each fp32 operation is the exact rational result rounded to
the nearest binary32 (ties to even)."""
from fractions import Fraction as F


def rn32(q):
    """Round a rational to the nearest fp32 (ties to even), as a Fraction.
    Normal range only (the emulated sequences keep every operand there)."""
    if q == 0:
        return F(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if F(2) ** e > a:
        e -= 1
    assert -126 <= e <= 127
    m = a / F(2) ** (e - 23)                    # in [2^23, 2^24)
    n = m.numerator // m.denominator
    r = m - n
    if r > F(1, 2) or (r == F(1, 2) and n % 2 == 1):
        n += 1
    return sign * F(n) * F(2) ** (e - 23)
