"""CPU check of the rounding argument the prefill rotation kernel rests on.

The kernel computes each rotated value x0 c - x1 s (and x0 s + x1 c) of bf16 inputs and FP64 angle
terms in FP32 (c, s rounded to FP32, one product and one fused multiply-add), bounds the FP32 error by
2^-23 (|x0| + |x1| + |y|) + 2^-149, and keeps the FP32 result when y minus and plus twice that bound
(again computed in FP32) round to the same bf16 value; otherwise it redoes the value in FP64.  The
claim: whenever the FP32 result is kept, its bf16 rounding is the bf16 rounding of the exact value.

Here every FP32 operation of that path is emulated exactly (rational arithmetic, one rounding to
nearest even per operation, subnormals kept), on random inputs and on inputs built to land next to a
bf16 rounding boundary, and each kept result is compared with the exact value's rounding.
"""
import math
import random
from fractions import Fraction

F32_MIN_EXP = -126   # smallest normal exponent of FP32 and bf16
F32_MANT = 23        # stored fraction bits of FP32
BF16_MANT = 7        # ... of bf16


def _floor_log2(a: Fraction) -> int:
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    return e


def _round(q: Fraction, mant: int) -> Fraction:
    """q rounded to nearest even in a binary format of `mant` fraction bits and FP32's exponent range."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = max(_floor_log2(a), F32_MIN_EXP)
    quantum = Fraction(2) ** (e - mant)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * quantum


def rn32(q: Fraction) -> Fraction:
    return _round(q, F32_MANT)


def rnbf16(q: Fraction) -> Fraction:
    return _round(q, BF16_MANT)


def kernel_component(x0: Fraction, x1: Fraction, c: float, s: float, second: bool):
    """(kept, bf16 value) of the kernel's FP32 path for x0 c - x1 s (second: x0 s + x1 c)."""
    cf, sf = rn32(Fraction(c)), rn32(Fraction(s))
    if not second:
        p = rn32(x1 * sf)
        y = rn32(x0 * cf - p)
    else:
        p = rn32(x1 * cf)
        y = rn32(x0 * sf + p)
    k22, k126 = Fraction(2) ** -22, Fraction(2) ** -126
    m = rn32(rn32(abs(x0) + abs(x1)) * k22 + k126)
    e = rn32(abs(y) * k22 + m)
    lo, hi = rn32(y - e), rn32(y + e)
    return rnbf16(lo) == rnbf16(hi), rnbf16(y)


def exact_component(x0: Fraction, x1: Fraction, c: float, s: float, second: bool) -> Fraction:
    C, S = Fraction(c), Fraction(s)
    return rnbf16(x0 * S + x1 * C if second else x0 * C - x1 * S)


def random_bf16(rng: random.Random, scale: float = 1.0) -> Fraction:
    return rnbf16(Fraction(rng.gauss(0.0, scale)))


def test_kept_results_round_like_the_exact_value():
    rng = random.Random(20240611)
    kept = redo = 0
    theta = 1.0e7
    for _ in range(6000):
        x0, x1 = random_bf16(rng), random_bf16(rng)
        pos = rng.randrange(0, 262144)
        f = theta ** (-rng.randrange(0, 64) / 64.0)
        a = pos * f
        c, s = math.cos(a), math.sin(a)
        for second in (False, True):
            ok, got = kernel_component(x0, x1, c, s, second)
            if ok:
                kept += 1
                assert got == exact_component(x0, x1, c, s, second), (x0, x1, c, s, second)
            else:
                redo += 1
    assert kept > 100 * max(redo, 1)  # the FP64 redo stays rare on ordinary inputs


def test_values_next_to_a_rounding_boundary_are_redone_or_exact():
    """x1 = 0, x0 bf16 and c chosen so that x0 c lies within a few FP64 ulps of a bf16 midpoint: the FP32
    rounding of c alone moves the product by up to 2^-24 relative, so the fast path must give way."""
    rng = random.Random(7)
    redone = 0
    for _ in range(3000):
        x0 = random_bf16(rng)
        if x0 == 0:
            continue
        lo_bf = random_bf16(rng, 0.5)
        if lo_bf == 0:
            continue
        e = max(_floor_log2(abs(lo_bf)), F32_MIN_EXP)
        mid = lo_bf + (1 if lo_bf > 0 else -1) * Fraction(2) ** (e - BF16_MANT - 1)
        target = mid * (1 + Fraction(rng.randint(-4, 4), 2 ** 52))
        c = float(target / x0)
        if not abs(c) <= 1.0:
            continue
        s = math.sqrt(max(0.0, 1.0 - c * c))
        for x1 in (Fraction(0), random_bf16(rng, 1e-3)):
            ok, got = kernel_component(x0, x1, c, s, False)
            if ok:
                assert got == exact_component(x0, x1, c, s, False), (x0, x1, c, s)
            else:
                redone += 1
    assert redone > 0


def test_rounding_helpers_against_known_values():
    # bf16 keeps 8 significant bits: 1 + 2^-8 is a tie between 1 and 1 + 2^-7 and goes to the even 1;
    # 1 + 3 * 2^-8 is a tie between 1 + 2^-7 and 1 + 2^-6 and goes to the even 1 + 2^-6
    assert rnbf16(1 + Fraction(1, 2 ** 8)) == 1
    assert rnbf16(1 + Fraction(3, 2 ** 8)) == 1 + Fraction(1, 2 ** 6)
    assert rnbf16(-(1 + Fraction(3, 2 ** 8))) == -(1 + Fraction(1, 2 ** 6))
    # FP32: 1 + 2^-24 ties to 1; the smallest subnormal is 2^-149 and half of it rounds to 0 (even)
    assert rn32(1 + Fraction(1, 2 ** 24)) == 1
    assert rn32(Fraction(1, 2 ** 149)) == Fraction(1, 2 ** 149)
    assert rn32(Fraction(1, 2 ** 150)) == 0
    assert rn32(Fraction(3, 2 ** 150)) == Fraction(2, 2 ** 149)
    # against numpy's float32 conversion on ordinary values
    import numpy as np

    rng = random.Random(3)
    for _ in range(2000):
        v = rng.gauss(0.0, 10.0) * 2.0 ** rng.randint(-30, 30)
        assert rn32(Fraction(v)) == Fraction(float(np.float32(v)))
