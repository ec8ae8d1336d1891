"""Exhaustive checks, in exact rational arithmetic, of the division scheme the CUDA
quantizers use for Eq. (1) of TwinQuant §2 (q_max = 7 for W4A4 activations and
weights, q_max = 127 for the W4A8 activations of §5.1).

The kernels never divide. With y = RN(1/b) (a constant for the scale, a correctly
rounded reciprocal for the codes), q0 = RN(a y) and r = RN(a - b q0) (one fma),
Markstein's correction q = RN(q0 + r y) is taken as the correctly rounded quotient
RN(a / b). These tests check that claim for every case the quantizers meet:
- scale: b = q_max, a any BF16 significand (powers of two scale out in the
  normal range);
- codes: b = s = RN(a / q_max), a and v BF16 with |v| <= a, every significand
  pair and every exponent offset at which the code can be nonzero.
They also check that the absmax itself always rounds to q_max, so the kernels
need no clamp.
"""
from fractions import Fraction as F

import pytest


def rn32(x: F) -> F:
    """Round a rational to the nearest float32 (normal range), ties to even."""
    if x == 0:
        return F(0)
    sign = -1 if x < 0 else 1
    x = abs(x)
    e = x.numerator.bit_length() - x.denominator.bit_length()
    if F(2) ** e > x:
        e -= 1
    ulp = F(2) ** (e - 23)
    k = x / ulp
    fl = k.numerator // k.denominator
    rem = k - fl
    if rem > F(1, 2) or (rem == F(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * ulp


def markstein(a: F, b: F, y: F) -> F:
    q0 = rn32(a * y)
    r = rn32(a - b * q0)
    return rn32(q0 + r * y)


BF16_SIGNIFICANDS = [F(m, 128) for m in range(128, 256)]  # [1, 2), 8 significant bits


@pytest.mark.parametrize("qmax", [7, 127])
def test_scale_step_is_correctly_rounded(qmax):
    y = rn32(F(1, qmax))
    for a in BF16_SIGNIFICANDS:
        assert markstein(a, F(qmax), y) == rn32(a / qmax), (qmax, a)


@pytest.mark.parametrize("qmax", [7, 127])
def test_code_quotient_is_correctly_rounded(qmax):
    # v / s >= 1/2 needs v >= a / (2 qmax): exponent offsets down to -(bits of 2 qmax)
    lowest = -((2 * qmax).bit_length())
    bad = []
    for a in BF16_SIGNIFICANDS:
        s = rn32(a / qmax)
        y = rn32(1 / s)
        assert markstein(a, s, y) == rn32(a / s)
        assert round(rn32(a / s)) == qmax  # the absmax maps to +-qmax: no clamp needed
        for e in range(lowest, 1):
            for vm in BF16_SIGNIFICANDS:
                v = vm * F(2) ** e
                if v > a:
                    continue
                if markstein(v, s, y) != rn32(v / s):
                    bad.append((a, v))
    assert not bad, bad[:4]
