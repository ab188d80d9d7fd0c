"""The quantizers' division-free quotient, checked in exact rational arithmetic.

The kernels never divide: per row they take R = RN(1/S) and Rlo =
RN(RN(1 - S R) R); per element q0 = RN(x R + RN(x Rlo)) and one FMA
correction q = RN(q0 + RN(x - q0 S) R) (Markstein's step from a faithful
first quotient).  The requantizing epilogue uses the scalar form with
q0 = RN(x R) and two corrections.  Here each operation is carried out on
Fractions and rounded to fp32 by hand (an FMA rounds once), and the result
is compared with the correctly rounded quotient RN(x / S), over scales from
absmax / 127 and absmax / 448, inputs on the fp32 and bf16 grids, and exact
rounding midpoints.  No GPU is involved.
"""
import math
import random
from fractions import Fraction as F

import numpy as np


def rn32(v: F) -> F:
    """v rounded to the nearest fp32 value, ties to even (normal and subnormal range)."""
    if v == 0:
        return F(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    while F(2) ** e > a:
        e -= 1
    while F(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    ulp = F(2) ** (e - 23)
    q = a / ulp
    n = q.numerator // q.denominator
    r = q - n
    if r > F(1, 2) or (r == F(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * ulp


def f32(x) -> F:
    return F(float(np.float32(x)))


def bf16(x) -> F:
    b = np.array([x], np.float32).view(np.uint32)[0]
    b = (int(b) + 0x7FFF + ((int(b) >> 16) & 1)) & 0xFFFF0000
    return F(float(np.array([b], np.uint32).view(np.float32)[0]))


def paired_quotient(x: F, S: F) -> F:
    R = rn32(1 / S)
    e = 1 - S * R
    assert rn32(e) == e            # 1 - S R is exact in an FMA
    Rlo = rn32(e * R)
    q0 = rn32(x * R + rn32(x * Rlo))
    return rn32(q0 + rn32(x - q0 * S) * R)


def scalar_quotient(x: F, S: F) -> F:
    R = rn32(1 / S)
    q0 = rn32(x * R)
    q1 = rn32(q0 + rn32(x - q0 * S) * R)
    return rn32(q1 + rn32(x - q1 * S) * R)


def _scales(rng):
    for i in range(24):
        amax = f32(rng.uniform(1e-3, 1e3) * (2.0 ** rng.randint(-20, 20)))
        yield amax, rn32(amax / (127 if i % 2 == 0 else 448))


def test_paired_and_scalar_quotients_are_correctly_rounded():
    rng = random.Random(3)
    n = 0
    for amax, S in _scales(rng):
        for _ in range(60):
            u = rng.uniform(-1.0, 1.0)
            for x in (f32(u * float(amax)), bf16(u * float(amax))):
                want = rn32(x / S)
                assert paired_quotient(x, S) == want, (x, S)
                assert scalar_quotient(x, S) == want, (x, S)
                n += 1
    assert n == 24 * 60 * 2


def test_quotients_on_rounding_midpoints():
    """x / S exactly on an integer midpoint (k + 1/2) and at absmax: the
    quotient must be exact there, or the rounding that follows moves."""
    rng = random.Random(5)
    for amax, S in _scales(rng):
        for k in (0, 1, 2, 62, 63, 100, 126):
            for x in (rn32((k + F(1, 2)) * S), -rn32((k + F(1, 2)) * S), amax, -amax):
                want = rn32(x / S)
                assert paired_quotient(x, S) == want
                assert scalar_quotient(x, S) == want


def test_first_quotient_alone_is_not_enough():
    """RN(x R) alone misses RN(x / S) for some inputs: the corrections are needed."""
    rng = random.Random(7)
    misses = 0
    for amax, S in _scales(rng):
        R = rn32(1 / S)
        for _ in range(200):
            x = f32(rng.uniform(-1.0, 1.0) * float(amax))
            misses += rn32(x * R) != rn32(x / S)
    assert misses > 0
