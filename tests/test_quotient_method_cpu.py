"""The division method of the inverse-RoPE + FP8 kernel, checked in exact
arithmetic on the CPU (no GPU, no kernel code).

The kernel forms each quotient y / s of its per-head quantisation without a
divide: with r = RN(1/s), n0 = RN(y * -r), e = RN(n0 * s + y) (one FMA, so
rounded once), n1 = RN(e * -r + n0) (one FMA), it takes -n1 as the correctly
rounded fp32 quotient (Markstein's theorem: P. Markstein, "Computation of
elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
Dev. 34(1), 1990), and the negated form keeps the sign of a zero quotient.
Here every step is evaluated exactly with rationals and rounded once to fp32
(round to nearest even), and -n1 is compared with RN(y / s) bit for bit,
including quotients that sit exactly on E4M3 rounding ties (where a one-ulp
error would change the 8-bit code) and signed zeros.
"""
import math
from fractions import Fraction as F

import numpy as np

FP32_MIN_EXP = -126


def rn32(x: F) -> float:
    """Round a rational to the nearest fp32 value, ties to even (normal and
    subnormal range; the inputs here never overflow)."""
    if x == 0:
        return 0.0
    neg = x < 0
    x = -x if neg else x
    e = x.numerator.bit_length() - x.denominator.bit_length()
    while F(2) ** e > x:
        e -= 1
    while F(2) ** (e + 1) <= x:
        e += 1
    e = max(e, FP32_MIN_EXP)
    ulp = F(2) ** (e - 23)
    m = x / ulp
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > F(1, 2) or (rem == F(1, 2) and fl % 2 == 1):
        fl += 1
    v = float(fl * ulp)
    return -v if neg else v


def fma_rn(a: float, b: float, c: float) -> float:
    """Fused multiply-add with one rounding, signed zero as IEEE 754 gives it."""
    exact = F(a) * F(b) + F(c)
    if exact == 0:
        p_neg = math.copysign(1.0, a) * math.copysign(1.0, b) < 0
        c_neg = math.copysign(1.0, c) < 0
        # x + y with both zero: -0 only when both are -0 (round to nearest)
        return -0.0 if (p_neg and c_neg) else 0.0
    return rn32(exact)


def mul_rn(a: float, b: float) -> float:
    exact = F(a) * F(b)
    if exact == 0:
        return -0.0 if math.copysign(1.0, a) * math.copysign(1.0, b) < 0 else 0.0
    return rn32(exact)


def quotient_by_method(y: float, s: float) -> float:
    r = rn32(F(1) / F(s))
    nr = -r
    n0 = mul_rn(y, nr)
    e = fma_rn(n0, s, y)
    n1 = fma_rn(e, nr, n0)
    return -n1


def quotient_exact(y: float, s: float) -> float:
    q = F(y) / F(s)
    if q == 0:
        return -0.0 if math.copysign(1.0, y) < 0 else 0.0
    return rn32(q)


def same_bits(a: float, b: float) -> bool:
    return np.float32(a).view(np.uint32) == np.float32(b).view(np.uint32)


def e4m3_ties():
    vals = sorted({(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8)}
                  | {m / 8 * 2.0 ** -6 for m in range(1, 8)})
    vals = [v for v in vals if v <= 448]
    return [(a + b) / 2 for a, b in zip(vals, vals[1:])]


def test_method_equals_correctly_rounded_division():
    rng = np.random.default_rng(17)
    ties = e4m3_ties()
    checked = 0
    for i in range(3000):
        # scales as the kernel forms them, fp32(amax) / 448, over a wide range
        s = float(np.float32(float(np.float32(rng.uniform(0.5, 2.0) * 10.0 ** rng.uniform(-20, 20))) / 448.0))
        if i % 3 == 0:   # quotients exactly on an E4M3 tie, or one fp32 ulp away
            q = ties[rng.integers(len(ties))] * rng.choice([-1.0, 1.0])
            y = float(np.float32(q * s))
            y = float(np.nextafter(np.float32(y), np.float32(np.inf) * rng.choice([-1, 1]))) if i % 6 == 3 else y
        else:
            y = float(np.float32(s * rng.uniform(-448.0, 448.0) * 10.0 ** rng.uniform(-6, 0)))
        got, want = quotient_by_method(y, s), quotient_exact(y, s)
        assert same_bits(got, want), (y, s, got, want)
        checked += 1
    assert checked == 3000


def test_zero_quotients_keep_the_sign_of_y():
    for s in (1.0, 3.0, 0.007, 5.5e-3, 2.0 ** -99):
        s = float(np.float32(s))
        for y in (0.0, -0.0):
            got, want = quotient_by_method(y, s), quotient_exact(y, s)
            assert same_bits(got, want), (y, s, got, want)
    # the plain order (q0 = RN(y r), e = RN(-q0 s + y), RN(e r + q0)) loses the sign of -0
    r = rn32(F(1) / F(3.0))
    q0 = mul_rn(-0.0, r)
    e = fma_rn(-q0, 3.0, -0.0)
    assert not same_bits(fma_rn(e, r, q0), -0.0)
