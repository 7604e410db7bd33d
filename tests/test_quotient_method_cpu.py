"""The quantisers' division method, checked in exact arithmetic on the CPU.

The GPU quantisers compute fl(x / s), the correctly rounded binary32
quotient, as y = RN(1/s), q = RN(x y) followed by two Markstein correction
steps q <- RN(q + RN(x - s q) y) (P. Markstein, IBM J. Res. Dev. 34, 1990),
and keep the sign of x.  Here every operation is emulated with exact
rationals and one rounding to binary32, and the result must equal the
correctly rounded quotient for random and adversarial operands (scale
mantissas of all ones, one, 2^22; bf16 and FP32 values up to 448 s)."""
from fractions import Fraction as F

import numpy as np


def rn32(fr):
    """A rational rounded to the nearest binary32, ties to even."""
    f = np.float32(float(fr))
    best = None
    for c in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
        d = abs(F(float(c)) - fr)
        if best is None or d < best[0] or (d == best[0] and int(np.float32(c).view(np.uint32)) % 2 == 0):
            best = (d, c)
    return np.float32(best[1])


def fma32(a, b, c):
    return rn32(F(float(a)) * F(float(b)) + F(float(c)))


def quotient(x, s):
    y = rn32(F(1) / F(float(s)))
    q = rn32(F(float(x)) * F(float(y)))
    q = fma32(fma32(-q, s, x), y, q)
    q = fma32(fma32(-q, s, x), y, q)
    return np.float32(np.copysign(q, x))


def operands(seed, n):
    rng = np.random.default_rng(seed)
    amax = (rng.random(n) * 10.0 ** rng.uniform(-6, 6, n)).astype(np.float32) + np.float32(1e-30)
    s = (amax / np.float32(448)).astype(np.float32)
    adv = rng.random(n) < 0.4
    mant = rng.choice([0x7FFFFF, 0x7FFFFE, 0x000001, 0x400000, 0x7FFF00], n)
    s = np.where(adv, (s.view(np.uint32) & 0xFF800000) | mant, s.view(np.uint32)).astype(np.uint32).view(np.float32)
    x = (rng.uniform(-1, 1, n).astype(np.float32) * s * np.float32(448)).astype(np.float32)
    xb = (x.view(np.uint32) & 0xFFFF0000).view(np.float32)
    return s, x, xb


def test_two_corrections_give_the_correctly_rounded_quotient():
    s, x, xb = operands(3, 6000)
    for xs in (x, xb):
        for xi, si in zip(xs, s):
            ref = rn32(F(float(xi)) / F(float(si)))
            got = quotient(xi, si)
            assert got == ref and np.signbit(got) == np.signbit(ref), (repr(xi), repr(si), repr(got), repr(ref))


def test_signed_zero_and_exact_quotients():
    for s in (np.float32(1.0), np.float32(0.75), np.float32(3.0) / np.float32(448)):
        assert np.signbit(quotient(np.float32(-0.0), s)) and quotient(np.float32(-0.0), s) == 0
        assert quotient(np.float32(0.0), s) == 0 and not np.signbit(quotient(np.float32(0.0), s))
        for k in (1, 3, 448):
            x = np.float32(s * np.float32(k))
            assert quotient(x, s) == rn32(F(float(x)) / F(float(s)))
