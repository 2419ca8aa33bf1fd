"""Pins for the oracle's per-token absmax int8 quantisation (CPU only).

The pages name BitNet b1.58's 8-bit activations (1bit.systems post "the full
arc ...", paper list item 1) without a formula. The reading under test:
s = fl32(127 / amax), q = clamp(rint(fl32(x * s)), -127, 127) with ties to
even, x_scale = fl32(amax / 127), x_sum = sum q; an all-zero row gives zeros.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from workloads import activations_bf16, bf16_bits_to_float
from tests._exact import bf16, round_half_even, round_to_fp32


def _row(vals):
    return np.array([[bf16(v) for v in vals]], dtype=np.uint16)


def test_hand_case_unit_amax():
    # amax = 1 -> s = 127 exactly; 1 -> 127; -0.5 -> -63.5 -> tie to even -64;
    # 0.25 -> 31.75 -> 32. x_sum = 127 - 64 + 32 = 95. x_scale = fl32(1/127).
    q, s, t = oracle.quant(_row([1.0, -0.5, 0.25]))
    assert q.tolist() == [[127, -64, 32]]
    assert t.tolist() == [95]
    assert s[0] == round_to_fp32(Fraction(1, 127))


def test_hand_case_amax_two():
    # amax = 2 -> s = 63.5 exactly. -2 -> -127; 1 -> 63.5 -> 64 (even);
    # 0.5 -> 31.75 -> 32; 0.75 -> 47.625 -> 48; -1.5 -> -95.25 -> -95.
    # x_sum = -127 + 64 + 32 + 48 - 95 = -78; x_scale = fl32(2/127).
    q, s, t = oracle.quant(_row([-2.0, 1.0, 0.5, 0.75, -1.5]))
    assert q.tolist() == [[-127, 64, 32, 48, -95]]
    assert t.tolist() == [-78]
    assert s[0] == round_to_fp32(Fraction(2, 127))


def test_zero_row():
    q, s, t = oracle.quant(np.zeros((2, 32), dtype=np.uint16))
    assert (q == 0).all() and (s == 0).all() and (t == 0).all()
    # negative zero is a zero too
    q, s, t = oracle.quant(np.full((1, 16), 0x8000, dtype=np.uint16))
    assert (q == 0).all() and s[0] == 0 and t[0] == 0


def _random_rows(M, K, seed):
    return activations_bf16(np.random.default_rng(seed), M, K)


@pytest.mark.parametrize("K", [16, 2560, 6912])
def test_invariants_random(K):
    M = 2000 if K <= 2560 else 400
    xb = _random_rows(M, K, K)
    x = bf16_bits_to_float(xb).astype(np.float64)
    q, s, t = oracle.quant(xb)
    qd = q.astype(np.float64)
    amax = np.abs(x).max(axis=1)
    # x_sum is the sum of the codes
    assert (t == q.astype(np.int64).sum(axis=1)).all()
    # the largest |x| maps to +-127 with its sign
    arg = np.abs(x).argmax(axis=1)
    assert (np.abs(q[np.arange(M), arg]) == 127).all()
    assert (np.sign(q[np.arange(M), arg]) == np.sign(x[np.arange(M), arg])).all()
    # sign preserved (a small |x| may round to 0)
    assert ((np.sign(qd) == np.sign(x)) | (q == 0)).all()
    # codes stay in [-127, 127]
    assert q.min() >= -127 and q.max() <= 127
    # x_scale is amax/127 to within one fp32 rounding
    assert np.all(np.abs(s.astype(np.float64) - amax / 127) <= amax / 127 * 2.0 ** -24)
    # reconstruction error: at most half a step (plus fp32 rounding slack)
    err = np.abs(qd * s[:, None].astype(np.float64) - x)
    assert np.all(err <= 0.5 * s[:, None] * (1 + 1e-4))


def test_negation_and_power_of_two_scaling():
    xb = _random_rows(500, 2560, 11)
    q, s, t = oracle.quant(xb)
    qn, sn, tn = oracle.quant(xb ^ np.uint16(0x8000))  # flip every sign bit
    assert (qn == -q).all() and (sn == s).all() and (tn == -t).all()
    # multiplying a row by 2 (exact in bf16: exponent + 1) keeps q and x_sum and
    # doubles x_scale exactly
    x2 = (bf16_bits_to_float(xb) * np.float32(2)).view(np.uint32) >> 16
    q2, s2, t2 = oracle.quant(x2.astype(np.uint16))
    assert (q2 == q).all() and (t2 == t).all() and (s2 == s * np.float32(2)).all()


def test_exact_rational_model():
    """Exact-rational restatement on random rows: the fp32 roundings, done with
    Fractions, give the same codes; and among them, rows where multiplying by
    fl32(127/amax) and dividing by fl32(amax/127) disagree confirm the former."""
    rng = np.random.default_rng(5)
    xb = activations_bf16(rng, 60, 256)
    q, s, t = oracle.quant(xb)
    x = bf16_bits_to_float(xb)
    for m in range(xb.shape[0]):
        amax = Fraction(float(np.abs(x[m]).max()))
        s32 = Fraction(float(round_to_fp32(Fraction(127) / amax)))
        for k in range(xb.shape[1]):
            xv = Fraction(float(x[m, k]))
            expect = round_half_even(Fraction(float(round_to_fp32(xv * s32))))
            expect = max(-127, min(127, expect))
            assert q[m, k] == expect, (m, k)


def test_random_against_float64_within_one_code():
    # A float64 statement of the same quantiser can differ only where fp32
    # rounding moved x*s across a half-integer: by one code, rarely.
    xb = _random_rows(20000, 64, 3)
    x = bf16_bits_to_float(xb).astype(np.float64)
    q, _, _ = oracle.quant(xb)
    amax = np.abs(x).max(axis=1, keepdims=True)
    ref = np.clip(np.rint(x * (127.0 / amax)), -127, 127)
    diff = np.abs(q - ref)
    assert diff.max() <= 1
    assert (diff > 0).mean() < 1e-4
