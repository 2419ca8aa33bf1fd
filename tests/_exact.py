"""Exact-arithmetic helpers for the oracle's pins (no oracle code here)."""
from fractions import Fraction
import math

import numpy as np


def round_to_fp32(v: Fraction) -> np.float32:
    """The fp32 value nearest to the rational v (ties to even), by exact arithmetic.
    Covers the normal range only, which is all the pins need."""
    if v == 0:
        return np.float32(0.0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    # fix e so that 2^e <= a < 2^(e+1)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 23)
    n = a / ulp                      # in [2^23, 2^24)
    lo = math.floor(n)
    rem = n - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return np.float32(sign * float(lo * ulp))


def round_half_even(v: Fraction) -> int:
    lo = math.floor(v)
    rem = v - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return int(lo)


def bf16(v: float) -> int:
    """bf16 bit pattern of a float that bf16 represents exactly (asserted)."""
    f = np.array([v], dtype=np.float32)
    u = int(f.view(np.uint32)[0])
    assert u & 0xFFFF == 0, f"{v} is not exactly representable in bf16"
    return u >> 16
