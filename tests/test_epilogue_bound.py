"""The fp32 rounding test of the W4A8 byte-plane GEMM's epilogue, checked in
exact rational arithmetic on the CPU.

Each output of that epilogue is y = sc * Y + bias with the exact integer
Y = A0 + 256 A1 + 65536 A2 (the digit sums; A2 = 0 without a top digit),
sc = sx 2^e_n and an fp32 bias.  The kernel forms, with one IEEE fp32
rounding per operation (conversions, fused multiply-adds, products, sums):

    a_p = fl(A_p);  yf = fma(a2, 65536, fma(a1, 256, a0))
    T   = fma(|a2|, 65536, fma(|a1|, 256, |a0|))
    v   = fma(sc, yf, bias)
    err = fma(fma(fl(1.5 sc), T, |v|), c1, c2),  c1 = 2^-23 (1 + 2^-16), c2 = 2^-99

and keeps bf16(v) when bf16(v - err) == bf16(v + err) (round to nearest even);
otherwise it recomputes the output in fp64.  Its claim: whenever the two
roundings agree, bf16(v) is the round-to-nearest-even bf16 of the exact y, and
the same bits as the fp64 path (one fp64 rounding of y, then bf16).  This test
emulates every fp32 step exactly (fractions, rounded to nearest even by
integer arithmetic) and checks that claim on random outputs, on outputs
placed within a few fp32 ulps of bf16 rounding midpoints, and on extreme
magnitudes; it also checks that the guard keeps most outputs on the fast path
(otherwise the test would pass vacuously)."""
from fractions import Fraction

import numpy as np

C1 = Fraction(1, 2 ** 23) * (1 + Fraction(1, 2 ** 16))
C2 = Fraction(1, 2 ** 99)


def ilog2(a: Fraction) -> int:
    """floor(log2(a)) for a > 0."""
    e = a.numerator.bit_length() - a.denominator.bit_length()
    return e - 1 if Fraction(2) ** e > a else e


def round_binary(q: Fraction, p: int, emin: int, emax: int):
    """q rounded to nearest even in a binary format with p significant bits,
    smallest normal exponent emin and largest exponent emax; returns a
    Fraction, or +-inf (as a float) on overflow."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = max(ilog2(a), emin)
    quantum = Fraction(2) ** (e - p + 1)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    r = fl * quantum
    if r >= Fraction(2) ** (emax + 1):
        return sign * float("inf")
    return sign * r


def f32(q):
    return round_binary(Fraction(q), 24, -126, 127)


def bf16(q):
    """Round-to-nearest-even bf16 of q, as (sign, value) so that -0 == +0 compare
    by value and infinities keep their sign."""
    r = round_binary(Fraction(q), 8, -126, 127) if not isinstance(q, float) else q
    return r


def fma(a, b, c):
    if any(isinstance(t, float) for t in (a, b, c)):  # an infinity on the way
        return float(a) * float(b) + float(c)
    return f32(a * b + c)


def fast_path(A, sc, bias):
    """The kernel's fp32 sequence; returns (kept, bf16 of v)."""
    a = [f32(x) for x in A]
    yf = fma(a[2], 65536, fma(a[1], 256, a[0]))
    T = fma(abs(a[2]), 65536, fma(abs(a[1]), 256, abs(a[0])))
    v = fma(sc, yf, bias)
    if isinstance(v, float):  # overflow: v - err and v + err cannot agree
        return False, None
    inner = fma(f32(Fraction(3, 2) * sc), T, abs(v))
    err = fma(inner, f32(C1), C2) if not isinstance(inner, float) else inner
    if isinstance(err, float):
        return False, None
    lo, hi = f32(v - err), f32(v + err)
    blo, bhi = bf16(lo), bf16(hi)
    return blo == bhi, bf16(v)


def exact_bf16(A, sc, bias):
    Y = A[0] + 256 * A[1] + 65536 * A[2]
    return bf16(sc * Y + bias)


def fp64_path_bf16(A, sc, bias):
    """The exact path: y rounded once to fp64, then to bf16."""
    Y = A[0] + 256 * A[1] + 65536 * A[2]
    return bf16(round_binary(sc * Y + bias, 53, -1022, 1023))


def check(A, sc, bias):
    kept, b = fast_path(A, sc, bias)
    if kept:
        want = exact_bf16(A, sc, bias)
        assert b == want, (A, sc, bias, b, want)
        assert fp64_path_bf16(A, sc, bias) == want, (A, sc, bias)
    return kept


def rand_case(rng, K=4096, top=True, bias_scale=0.1):
    # digit sums of a realistic size (xq ~ 26 rms, digits ~ 74 rms over K)
    s = np.sqrt(K) * 26 * 74
    A = [int(rng.normal(0, s)), int(rng.normal(0, s / 4)), int(rng.normal(0, 3000)) if top else 0]
    sx = f32(Fraction(float(rng.uniform(0.01, 0.05))))
    sc = sx * Fraction(2) ** int(rng.integers(-24, -10))
    bias = f32(Fraction(float(rng.normal(0, bias_scale))))
    return A, sc, bias


def test_random_outputs_match_the_exact_rounding():
    rng = np.random.default_rng(1)
    kept = sum(check(*rand_case(rng, top=bool(i % 3 == 0))) for i in range(3000))
    assert kept > 2900  # the guard keeps almost every output on the fast path


def test_outputs_near_bf16_midpoints():
    """Biases chosen so that y lands within a few fp32 ulps of a bf16 rounding
    midpoint, on either side: the guard must send these to the exact path or
    get them right.  The bias is a quarter of the product (the product's
    rounding dominates the error) or a thousand times it (the rounding of v
    does)."""
    rng = np.random.default_rng(2)
    kept = 0
    for i in range(6000):
        A, sc, _ = rand_case(rng, top=bool(i % 2))
        p = sc * (A[0] + 256 * A[1] + 65536 * A[2])
        # a bf16 midpoint near 1.25 p or 1001 p
        target = f32((Fraction(5, 4) if i % 4 < 2 else Fraction(1001)) * p)
        if target == 0:
            continue
        b = round_binary(target, 8, -126, 127)
        e = ilog2(abs(b))
        mid = b + (Fraction(2) ** (e - 8) if b > 0 else -Fraction(2) ** (e - 8))
        ulp32 = Fraction(2) ** (e - 23)
        delta = int(rng.integers(-6, 7)) * ulp32 / int(rng.choice([1, 2, 4]))
        bias = f32(mid - p + delta)
        kept += check(A, sc, bias)
    assert kept > 0


def test_extreme_magnitudes():
    rng = np.random.default_rng(3)
    cases = []
    big = 127 * 128 * 65536  # |A_p| at K = 65536
    for _ in range(400):
        A = [int(rng.integers(-big, big)), int(rng.integers(-big, big)), int(rng.integers(-big, big))]
        ex = int(rng.integers(-124, 100))
        sc = f32(Fraction(float(rng.uniform(1, 2)))) * Fraction(2) ** ex
        bias = f32(Fraction(float(rng.normal(0, 1))) * Fraction(2) ** int(rng.integers(-140, 120)))
        cases.append((A, sc, bias))
    # cancellation between the planes (signed digits), tiny results, zero Y
    cases += [([5, -1, 0], Fraction(2) ** -124, Fraction(0)),
              ([256, -1, 0], Fraction(2) ** -100, f32(Fraction(1, 10 ** 30))),
              ([0, 0, 0], Fraction(1, 64), f32(Fraction(1, 3))),
              ([-65536, 0, 1], Fraction(2) ** 10, Fraction(0)),
              ([big, big, big], Fraction(2) ** 100, Fraction(0))]
    for A, sc, bias in cases:
        check(A, sc, bias)


def test_cancellation_between_planes():
    """Digit sums whose weighted terms nearly cancel (|256 A1| and |65536 A2|
    far above |Y|, A1 beyond fp32's exact integers): the conversion errors
    scale with T, not with |Y|, so a bound in |yf| alone would keep wrong
    results here."""
    rng = np.random.default_rng(5)
    for _ in range(1500):
        k = int(rng.integers(2 ** 17, 2 ** 22))
        A = [int(rng.integers(-2 ** 20, 2 ** 20)), 256 * k + int(rng.integers(-255, 256)), -k]
        sc = f32(Fraction(float(rng.uniform(1, 2)))) * Fraction(2) ** int(rng.integers(-30, -10))
        bias = f32(Fraction(float(rng.normal(0, 1e-3))))
        check(A, sc, bias)


def test_the_rounding_helpers():
    # pins of the emulation itself against numpy's IEEE fp32 and known values
    rng = np.random.default_rng(4)
    for _ in range(200):
        x, y = (np.float32(v) for v in rng.normal(0, 1e3, 2))
        assert f32(Fraction(float(x)) * Fraction(float(y))) == Fraction(float(x * y))
        assert f32(Fraction(float(x)) + Fraction(float(y))) == Fraction(float(x + y))
    assert round_binary(Fraction(1) + Fraction(1, 2 ** 8), 8, -126, 127) == 1  # tie to even
    assert round_binary(Fraction(1) + Fraction(3, 2 ** 8), 8, -126, 127) == 1 + Fraction(1, 64)
    assert round_binary(Fraction(2) ** 128, 24, -126, 127) == float("inf")
    assert round_binary(Fraction(3, 2 ** 150), 24, -126, 127) == Fraction(2, 2 ** 149)
