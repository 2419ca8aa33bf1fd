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


# ------------------------------------------------ order-free fp64 statistics
# The RMSNorm factor and the absmean scale are fp64 sums rounded to fp32
# after a few more fp64 operations. The GPU adds in a tree order, the oracle
# left to right; both results lie within (n - 1) u S of the exact sum S of
# the n non-negative terms (u = 2^-53; each term x^2 of an fp32 x, or |x| of a
# bf16 x, is exact in fp64). The operations after the sum are the same IEEE
# operations on both sides and are monotone in the sum, so if both ends of
# that interval give the same fp32 result, every order of the additions does.

U64 = 2.0 ** -53


def rms_factor(S: float, K: int, eps32: float) -> np.float32:
    """fl32(1 / sqrt(S / K + eps)) with the fp64 operations of the oracle."""
    return np.float32(1.0 / math.sqrt(S / K + eps32))


def rms_interval_ok(S: float, K: int, eps32: float) -> bool:
    """True if every sum within the order-error band around S (K terms)
    gives the same fp32 factor."""
    d = K * U64 * S * 1.0000001                       # (n - 1) u S, and the rounding of S
    return rms_factor(max(S - d, 0.0), K, eps32) == rms_factor(S + d, K, eps32)


def rms_order_free(v: np.ndarray, eps: float) -> np.ndarray:
    """Per row of fp32 v [M, K]: True if every fp64 summation order of the
    squares gives the same fp32 RMSNorm factor."""
    v = np.asarray(v, np.float32)
    eps32 = float(np.float32(eps))
    M, K = v.shape
    out = np.empty(M, bool)
    for m in range(M):
        sq = (v[m].astype(np.float64)) ** 2           # exact squares
        out[m] = rms_interval_ok(math.fsum(sq.tolist()), K, eps32)  # exactly rounded sum
    return out


def absmean_order_free(w_bits: np.ndarray) -> bool:
    """True if every fp64 summation order of |W| (bf16 bit patterns) gives
    the same fp32 scale fl32(S / n)."""
    a = np.abs((w_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)).ravel()
    n = a.size
    if n == 0:
        return True
    S = math.fsum(a.tolist())
    d = n * U64 * S * 1.0000001
    return np.float32(max(S - d, 0.0) / n) == np.float32((S + d) / n)
