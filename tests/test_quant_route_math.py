"""Exhaustive CPU checks of the two arithmetic facts the GPU quantizers' fast
route rests on (the device check, flexq_debug_check_quantizer, runs the route
itself on every (x, s, Q)):

1. RN32(a / Q) = fma(fma(-q0, Q, a), rq, q0) with q0 = RN32(a * rq) and
   rq = RN32(1 / Q), for every positive finite FP16 a and Q in {31, 127}:
   the scale needs no division.
2. A normal FP16 scale s = fp16(RN32(amax / Q)) bounds amax / s below
   Q + 1/2: inside a group with such a scale no code needs the clamp, and the
   rounding addend 1.5 * 2^23 stays exact (|x / s| far below 2^22).

All arithmetic here is exact (Python rationals, rounded to FP32 by hand)."""

from fractions import Fraction

import numpy as np
import pytest


def rn32(fr):
    """A rational rounded to the nearest FP32 value, ties to even (no
    overflow or FP32 subnormals occur in these checks)."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    fr = abs(fr)
    e = fr.numerator.bit_length() - fr.denominator.bit_length()
    while Fraction(2) ** e > fr:
        e -= 1
    while Fraction(2) ** (e + 1) <= fr:
        e += 1
    assert e >= -126
    ulp = Fraction(2) ** (e - 23)
    n = fr / ulp
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * ulp


def fp16_positive_finite():
    return np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)


def test_rn32_rounds_like_numpy():
    rng = np.random.default_rng(0)
    for v in rng.standard_normal(2000) * 10.0 ** rng.integers(-20, 20, 2000):
        assert float(rn32(Fraction(float(v)))) == float(np.float32(v))
    assert rn32(Fraction(1) + Fraction(1, 2 ** 24)) == 1                  # tie to even
    assert rn32(Fraction(1) + Fraction(3, 2 ** 24)) == 1 + Fraction(1, 2 ** 22)


@pytest.mark.parametrize("Q", [31, 127])
def test_scale_without_division_is_the_ieee_quotient(Q):
    rq = rn32(Fraction(1, Q))
    bad = []
    for a in fp16_positive_finite():
        A = Fraction(float(a))
        q0 = rn32(A * rq)
        r = rn32(A - q0 * Q)              # fma(-q0, Q, a): one rounding
        q1 = rn32(r * rq + q0)            # fma(r, rq, q0): one rounding
        if q1 != rn32(A / Q):
            bad.append(float(a))
    assert not bad, bad[:5]


@pytest.mark.parametrize("Q", [31, 127])
def test_normal_scales_keep_quotients_below_q_plus_half(Q):
    a = fp16_positive_finite()
    s32 = (a.astype(np.float32) / np.float32(Q)).astype(np.float32)     # IEEE FP32 division
    s16 = s32.astype(np.float16).astype(np.float64)
    normal = s16 >= 2.0 ** -14
    assert normal.sum() > 20000
    assert np.all(a[normal] / s16[normal] < Q + 0.5)
