"""Markstein's correction of a reciprocal product, checked in exact arithmetic.

The GPU quantizers form the IEEE fp32 quotient RN(x / delta), on which the INT8 and
E4M3 codes are defined, as RN(q + r y), with y = RN(1 / delta), q = RN(x y) and
r = RN(x - q delta), the remainder taken exactly in one fma (P. Markstein, "Computation
of elementary functions on the IBM RISC System/6000 processor", IBM J. Res. Develop. 34,
1990).  Here each fp32 rounding is carried out on exact rationals, and the result is
compared with the correctly rounded quotient: on random scales and inputs, and on inputs
placed within a few ulps of INT8 half-integers and of E4M3 rounding boundaries, where a
plain product x * y can round to the wrong code.  The GPU side is
tests/test_gpu_quotient.py.
"""
from fractions import Fraction as Fr
import random

import numpy as np


def rn32(v: Fr) -> np.float32:
    """v rounded to the nearest fp32 (ties to even), v within the normal range."""
    c = np.float32(float(v))
    best = None
    for cand in (np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))):
        key = (abs(Fr(float(cand)) - v), int(np.float32(cand).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return np.float32(best[1])


def markstein(x: np.float32, delta: np.float32) -> np.float32:
    y = rn32(Fr(1) / Fr(float(delta)))
    q = rn32(Fr(float(x)) * Fr(float(y)))
    r = rn32(Fr(float(x)) - Fr(float(q)) * Fr(float(delta)))
    return rn32(Fr(float(q)) + Fr(float(r)) * Fr(float(y)))


def _cases():
    rng = random.Random(4242)
    out = []
    for _ in range(600):   # random scales and inputs within the group's range
        delta = np.float32(2.0 ** rng.uniform(-40, 40) * (1 + rng.random()))
        x = np.float32(rng.uniform(-1, 1) * 127.0 * float(delta))
        out.append((x, delta))
    for _ in range(600):   # inputs next to INT8 half-integers k + 1/2
        delta = np.float32(2.0 ** rng.uniform(-30, 30) * (1 + rng.random()))
        k = rng.randint(-127, 126)
        x = rn32(Fr(2 * k + 1, 2) * Fr(float(delta)))
        for _ in range(rng.randint(0, 3)):
            x = np.nextafter(x, np.float32(rng.choice([-np.inf, np.inf])))
        out.append((np.float32(x), delta))
    for _ in range(600):   # inputs next to E4M3 rounding boundaries (midpoints of adjacent codes)
        delta = np.float32(2.0 ** rng.uniform(-30, 30) * (1 + rng.random()))
        e = rng.randint(-6, 7)
        m = rng.randint(0, 7)
        mid = Fr(2) ** e * (1 + Fr(2 * m + 1, 16))   # between 2^e (1 + m/8) and 2^e (1 + (m+1)/8)
        x = rn32(mid * Fr(float(delta)) * rng.choice([-1, 1]))
        for _ in range(rng.randint(0, 3)):
            x = np.nextafter(x, np.float32(rng.choice([-np.inf, np.inf])))
        out.append((np.float32(x), delta))
    return out


def test_markstein_quotient_is_the_correctly_rounded_quotient():
    bad = [(x, d) for x, d in _cases() if markstein(x, d) != rn32(Fr(float(x)) / Fr(float(d)))]
    assert not bad, "%d mismatches, e.g. x=%r delta=%r" % (len(bad), *bad[0])


def test_plain_product_misrounds_some_of_these_cases():
    """The check has teeth: RN(x * RN(1 / delta)) alone differs from the correctly rounded
    quotient on some of the constructed near-tie inputs."""
    diff = 0
    for x, d in _cases():
        y = rn32(Fr(1) / Fr(float(d)))
        if rn32(Fr(float(x)) * Fr(float(y))) != rn32(Fr(float(x)) / Fr(float(d))):
            diff += 1
    assert diff > 0
