"""The reconstruction table's division, checked on the CPU in exact arithmetic.

The kernels build W_hat_k = (k - z)/s as q0 = RN(a y) with y = RN(1/s) and a = RN(k - z), then
apply two remainder corrections q <- RN(q + RN(a - s q) y), each inner and outer step a single
fused multiply-add (one rounding of an exact value).  By Markstein's theorem (IBM J. Res. Dev.
34(1), 1990) the second correction returns RN(a/s) once the first has brought q within one ulp.
Here every step is computed exactly with rationals and rounded to binary32 by hand, and the
result is compared with the correctly rounded quotient.  The inputs follow the kernel's range
guard: |z| >= 2^-60 or z = 0, and 2^-60 <= s <= 2^30.
"""
from fractions import Fraction

import numpy as np
import pytest


def rn32(x: Fraction) -> Fraction:
    """x rounded to the nearest binary32 value, ties to even (normal range only)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    elif Fraction(2) ** (e + 1) <= a:
        e += 1
    assert -126 <= e <= 127, "outside the normal range"
    m = a / Fraction(2) ** (e - 23)          # in [2^23, 2^24)
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * Fraction(fl) * Fraction(2) ** (e - 23)


def f32(v: float) -> Fraction:
    return Fraction(float(np.float32(v)))


def table_entry(k: int, s: Fraction, z: Fraction) -> Fraction:
    y = rn32(1 / s)
    a = rn32(Fraction(k) - z)
    if a == 0:
        return Fraction(0)
    q = rn32(a * y)
    for _ in range(2):
        r = rn32(a - s * q)
        q = rn32(q + r * y)
    return q


def cases():
    r = np.random.default_rng(2024)
    out = []
    for _ in range(6000):
        s = f32(10.0 ** r.uniform(-4.6, 4.3))                  # the scales min-max gives
        z = f32(r.uniform(-40, 40))
        out.append((int(r.integers(0, 16)), s, z))
    for _ in range(1500):                                      # divisors 1.111...1 x 2^e
        e = int(r.integers(-12, 14))
        s = Fraction((1 << 24) - 1, 1 << 23) * Fraction(2) ** e
        out.append((int(r.integers(0, 16)), s, f32(r.uniform(-20, 20))))
    for _ in range(1500):                                      # z near a code value
        k = int(r.integers(0, 16))
        z = f32(k + float(r.choice([-1, 1])) * 2.0 ** -float(r.integers(5, 22)))
        out.append((k, f32(10.0 ** r.uniform(-3, 4)), z))
    for _ in range(500):                                       # tiny zeros at the guard's edge
        out.append((int(r.integers(0, 16)), f32(10.0 ** r.uniform(-2, 4)),
                    f32(float(r.choice([-1, 1])) * 2.0 ** -float(r.integers(40, 60)))))
    return out


@pytest.mark.parametrize("chunk", range(4))
def test_two_corrections_give_the_correctly_rounded_quotient(chunk):
    cs = cases()
    n = len(cs) // 4
    for k, s, z in cs[chunk * n:(chunk + 1) * n]:
        want = rn32(rn32(Fraction(k) - z) / s)
        got = table_entry(k, s, z)
        assert got == want, (k, float(s), float(z), float(got), float(want))
