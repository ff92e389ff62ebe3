"""The fp32 path of the W8A8 GEMM's epilogue, checked in exact rational
arithmetic on the CPU.

Each output is y = acc sx sw + bias (acc the exact int32 sum, sx, sw, bias
fp32).  The kernel forms r = fma(fl(fl(acc) sx), sw, bias) with one IEEE fp32
rounding per operation and keeps bf16(r) when acc == 0 or
|r| >= max(2^-12 |bias|, 2^-100); other outputs take the exact fp64 path.  Its
claim: the kept value's error is at most 2^-23 |acc sx sw| + 2^-24 |r|, under an
eighth of a bf16 ulp, so bf16(r) is within one bf16 ulp of the exact y rounded
once (the 2-ulp contract with the oracle).  This test emulates the fp32 steps
exactly (fractions rounded to nearest even) and checks both the error bound
and the ulp distance on random outputs, outputs whose bias cancels most of the
product, and a range of magnitudes of the scales (activation scales down to
the smallest the quantizer produces); it also checks that the guard keeps
most outputs on the fast path."""
from fractions import Fraction

import numpy as np

from .test_epilogue_bound import f32, fma, round_binary

GUARD = Fraction(1, 2 ** 12)
TINY = Fraction(1, 2 ** 100)


def bf16_ordinal(q):
    """A monotone integer for the round-to-nearest-even bf16 of q (finite)."""
    r = round_binary(Fraction(q), 8, -126, 127)
    assert not isinstance(r, float)
    if r == 0:
        return 0
    a = abs(r)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)
    code = int(a / Fraction(2) ** (e - 7)) + (e + 126) * 128  # monotone in |r|
    return code if r > 0 else -code


def fast_path(acc, sx, sw, bias):
    """(kept, r): the kernel's fp32 value and whether its guard keeps it."""
    p = f32(f32(acc) * sx)
    r = fma(p, sw, bias)
    if isinstance(r, float):
        return False, None
    z = max(f32(GUARD * abs(bias)), TINY)
    return (acc == 0 or abs(r) >= z), r


def check(acc, sx, sw, bias):
    kept, r = fast_path(acc, sx, sw, bias)
    if kept:
        y = acc * sx * sw + bias
        bound = Fraction(1, 2 ** 23) * abs(acc * sx * sw) + Fraction(1, 2 ** 24) * abs(r)
        assert abs(r - y) <= bound, (acc, sx, sw, bias)
        assert abs(bf16_ordinal(r) - bf16_ordinal(y)) <= 1, (acc, sx, sw, bias)
    return kept


def rand_scales(rng, sx_exp=(-24, 0)):
    sx = f32(Fraction(float(rng.uniform(0.5, 1.0))) * Fraction(2) ** int(rng.integers(*sx_exp)))
    sw = f32(Fraction(float(rng.uniform(0.5, 1.0))) * Fraction(2) ** int(rng.integers(-20, 0)))
    return sx, sw


def test_random_outputs():
    rng = np.random.default_rng(11)
    kept = 0
    for _ in range(3000):
        K = int(rng.choice([256, 3072, 12288]))
        acc = int(rng.normal(0, np.sqrt(K) * 40 * 40))
        sx, sw = rand_scales(rng)
        scale = abs(acc * sx * sw) or Fraction(1)
        bias = f32(Fraction(float(rng.normal(0, 1))) * scale)
        kept += check(acc, sx, sw, bias)
    assert kept > 2700


def test_bias_cancelling_the_product():
    rng = np.random.default_rng(12)
    for _ in range(3000):
        acc = int(rng.integers(-127 * 127 * 4096, 127 * 127 * 4096))
        sx, sw = rand_scales(rng)
        p = acc * sx * sw
        rel = Fraction(float(rng.uniform(-1, 1))) * Fraction(2) ** int(rng.integers(-30, 0))
        bias = f32(-p * (1 + rel))
        check(acc, sx, sw, bias)


def test_small_activation_scales():
    """Activation scales down to 2^-126 (the quantizer's smallest): products
    near the fp32 underflow go to the exact path, the kept ones hold."""
    rng = np.random.default_rng(13)
    for _ in range(1500):
        acc = int(rng.integers(-127 * 127 * 4096, 127 * 127 * 4096))
        sx, sw = rand_scales(rng, sx_exp=(-126, -60))
        bias = f32(Fraction(float(rng.normal(0, 1))) * (abs(acc * sx * sw) or Fraction(1)))
        check(acc, sx, sw, bias)


def test_extremes():
    big = 127 * 127 * 65536
    cases = [(0, Fraction(1, 3), Fraction(1, 7), f32(Fraction(1, 3))),
             (1, Fraction(2) ** -126, Fraction(2) ** -20, Fraction(0)),
             (big, Fraction(2) ** -20, Fraction(2) ** -20, Fraction(0)),
             (-big, Fraction(1, 127), Fraction(1, 127), f32(Fraction(10 ** 6))),
             (3, Fraction(2) ** -126, Fraction(1), f32(Fraction(2) ** -110))]
    for acc, sx, sw, bias in cases:
        check(acc, f32(sx), f32(sw), bias)


GUARD_GATE = Fraction(1, 2 ** 13)


def gated_fast_path(acc, sx, sw, bias, gate, res):
    """The gated epilogue's fp32 sequence: u = fma(fl(fl(acc) sx), sw, bias),
    y = fma(gate, u, residual), kept when |y| >= fma(2^-13 |gate|, |u| + |bias|,
    2^-100) (each step one fp32 rounding)."""
    u = fma(f32(f32(acc) * sx), sw, bias)
    y = fma(gate, u, res)
    if isinstance(y, float) or isinstance(u, float):
        return False, None
    z = fma(f32(GUARD_GATE * abs(gate)), f32(abs(u) + abs(bias)), TINY)
    return abs(y) >= z, y


def check_gated(acc, sx, sw, bias, gate, res):
    kept, y32 = gated_fast_path(acc, sx, sw, bias, gate, res)
    if kept:
        y = gate * (acc * sx * sw + bias) + res
        assert abs(bf16_ordinal(y32) - bf16_ordinal(y)) <= 1, (acc, sx, sw, bias, gate, res)
    return kept


def bf16_value(v: float) -> Fraction:
    return round_binary(Fraction(float(v)), 8, -126, 127)


def test_gated_outputs():
    """The gated residual epilogue y = residual + gate (acc sx sw + bias):
    random outputs and residuals that cancel most of the update."""
    rng = np.random.default_rng(14)
    kept = 0
    for i in range(4000):
        acc = int(rng.normal(0, 64 * 40 * 40))
        sx, sw = rand_scales(rng)
        u = acc * sx * sw
        bias = f32(Fraction(float(rng.normal(0, 1))) * (abs(u) or Fraction(1)))
        gate = f32(Fraction(float(rng.normal(0, 0.5))))
        if i % 2:
            res = bf16_value(float(rng.normal(0, 1)) * float(abs(u + bias) or 1))
        else:  # the residual cancels the update to a small relative remainder
            rel = Fraction(float(rng.uniform(-1, 1))) * Fraction(2) ** int(rng.integers(-20, 0))
            res = bf16_value(float(-gate * (u + bias) * (1 + rel)))
        kept += check_gated(acc, sx, sw, bias, gate, res)
    assert kept > 2000
