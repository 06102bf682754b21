"""The NVFP4 kernels form fl(x / S) without a division: y = fl(1/S), then
q0 = fl(x y), q1 = fl(q0 + fl(x - S q0) y), q2 = fl(q1 + (x - S q1) y) with
fused multiply-adds (Markstein, IBM J. Res. Dev. 34(1), 1990).  This CPU test
replays that sequence in exact rational arithmetic (an exact FMA and an exact
binary32 round-to-nearest-even) and checks q2 == fl(x / S) on random and
adversarial operands: exact E2M1 ties x = m S, their 1-ulp neighbours, and
random significands across binades.  No GPU and no oracle code involved."""
from fractions import Fraction
import random

import numpy as np

EMIN, P = -126, 24            # binary32: smallest normal exponent, precision


def rn32(v: Fraction) -> Fraction:
    """Exact round-to-nearest-even of a rational to binary32 (finite range)."""
    if v == 0:
        return Fraction(0)
    s = -1 if v < 0 else 1
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    q = max(e, EMIN) - (P - 1)                 # quantum exponent (subnormals keep EMIN - 23)
    scaled = a / (Fraction(2) ** q)
    n, r = divmod(scaled.numerator, scaled.denominator)
    rem = Fraction(r, scaled.denominator)
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return s * Fraction(n) * Fraction(2) ** q


def f32(x: float) -> Fraction:
    return Fraction(float(np.float32(x)))


def fma(a, b, c):
    return rn32(a * b + c)


def quotient_chain(x: Fraction, S: Fraction) -> Fraction:
    y = rn32(1 / S)
    q = rn32(x * y)
    q = fma(fma(-q, S, x), y, q)
    return fma(fma(-q, S, x), y, q)


def _cases():
    rng = random.Random(20260)
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    for _ in range(1500):                                   # random significands and binades
        S = f32(rng.uniform(1, 2) * 2.0 ** rng.randint(-60, 60))
        x = f32(rng.uniform(-7, 7) * float(S))
        yield x, S
    for _ in range(400):                                    # exact ties x = m S and 1-ulp neighbours
        S = f32(rng.choice([1.0, 1.5, 1.25, 1.75]) * 2.0 ** rng.randint(-20, 20))
        m = rng.choice(mids) * rng.choice([1, -1])
        x = Fraction(m) * S
        if rn32(x) != x:
            continue
        up = Fraction(float(np.nextafter(np.float32(float(x)), np.float32(np.inf))))
        dn = Fraction(float(np.nextafter(np.float32(float(x)), np.float32(-np.inf))))
        yield x, S
        yield up, S
        yield dn, S
    for _ in range(400):                                    # long-significand S near ties
        S = f32(rng.uniform(1, 2))
        m = rng.choice(mids)
        x = rn32(Fraction(m) * S)
        yield x, S


def test_division_free_quotient_equals_ieee_division():
    n = 0
    for x, S in _cases():
        want = rn32(x / S)
        got = quotient_chain(x, S)
        assert got == want, (float(x), float(S), float(got), float(want))
        n += 1
    assert n > 2500


def test_one_correction_is_not_always_enough_in_theory():
    """q0 alone can miss by an ulp (it is why the chain corrects twice):
    find such a case among random operands."""
    rng = random.Random(7)
    misses = 0
    for _ in range(3000):
        S = f32(rng.uniform(1, 2))
        x = f32(rng.uniform(1, 2))
        if rn32(x * rn32(1 / S)) != rn32(x / S):
            misses += 1
    assert misses > 0


def _sr_up(v: Fraction, u24: int) -> bool:
    """The stochastic decision between 0 and 0.5 for |v| < 0.5: up iff
    u < |v| / 0.5 with u = u24 * 2^-24."""
    return Fraction(u24, 1 << 24) < abs(v) / Fraction(1, 2)


def test_underflowing_quotients_decide_the_same_codes():
    """Markstein's theorem assumes no underflow, but the kernels use the chain
    for every S in [2^-125, 2^125], so x / S may be subnormal (a block whose
    values span more than 2^126).  There the chain can miss fl(x / S) by an
    ulp; this pins that every such miss is harmless: both results have the
    same sign and the same zero-ness, and both lie far below 2^-25, where the
    E2M1 nearest code is a signed zero and the stochastic decision between 0
    and 0.5 depends only on whether v is zero (u is a multiple of 2^-24)."""
    rng = random.Random(31)
    n = misses = 0
    for _ in range(6000):
        S = f32(rng.uniform(1, 2) * 2.0 ** rng.randint(-125, 125))
        e = rng.randint(-172, -110)
        x = rn32(Fraction(rng.uniform(1, 2)) * Fraction(2) ** e * S) * rng.choice([1, -1])
        want = rn32(x / S)
        got = quotient_chain(x, S)
        n += 1
        if got == want:
            continue
        misses += 1
        assert (got == 0) == (want == 0) and (got < 0) == (want < 0), (float(x), float(S))
        assert max(abs(got), abs(want)) < Fraction(1, 1 << 100), (float(x), float(S))
        for u24 in (0, 1, (1 << 24) - 1):
            assert _sr_up(got, u24) == _sr_up(want, u24)
    assert n > 5000 and misses > 0           # the underflow range really is exercised
