"""The algebra behind the W4A8 GEMM route, checked in exact arithmetic on the CPU.

For weight row n with fp16 scales s[n,g] and offsets o[n,g], let e_n be the
smallest exponent of the lowest set bit over the row's nonzero values.  Then
S = s / 2^e_n and O = o / 2^e_n are integers, every dequantized weight s q + o
is 2^e_n W with the integer W = S q + O, and the per-group fold equals
2^e_n Y with the integer GEMM Y = sum_k xq W.  When U = W + 0x80..80 fits P
bytes, W = sum_p 256^p d_p with the signed digits d_p = U_p - 128 in
[-128, 127], so Y is P int8 GEMMs on the digits.  The route rounds
sx 2^e_n Y + bias once to bf16.

This test computes all of that with Python integers and fractions (nothing
of the library, nothing of its kernels): the grid (every weight and every
fold term exactly reproduced), the digits, the digit GEMMs, and the single
rounding.  It compares that rounding with the oracle's output, which rounds
its fp64 fold: they agree bit for bit wherever the fold is exact in fp64, and
within one bf16 ulp anywhere.  Weights: Gaussian through the oracle's
quantizer (two or three digits), integer-valued groups (one digit), and rows
with one group of subnormal fp16 scale and offset (three digits)."""
from fractions import Fraction

import numpy as np

import oracle
from w4a8_quantized_gemm_token_b200 import synthetic

from .helpers import bf16_ulp_distance


def f16_value(bits: int) -> Fraction:
    """The exact value of an fp16 bit pattern (finite)."""
    sign = -1 if bits & 0x8000 else 1
    e = (bits >> 10) & 31
    m = bits & 1023
    assert e != 31
    if e == 0:
        return sign * Fraction(m, 2 ** 24)
    return sign * Fraction(1024 + m, 2 ** 10) * Fraction(2) ** (e - 15)


def lowest_bit_exponent(v: Fraction) -> int:
    """The exponent of the lowest set bit of a nonzero dyadic rational."""
    num, den = abs(v.numerator), v.denominator
    assert den & (den - 1) == 0
    tz = (num & -num).bit_length() - 1
    return tz - (den.bit_length() - 1)


def bf16_rne(q: Fraction) -> int:
    """Round-to-nearest-even bf16 bits of an exact value (finite, normal range)."""
    if q == 0:
        return 0
    sign = 0x8000 if q < 0 else 0
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    assert -126 <= e <= 127
    quantum = Fraction(2) ** (e - 7)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    value = fl * quantum  # may carry into the next binade: still exact in bf16
    e2 = value.numerator.bit_length() - value.denominator.bit_length()
    if Fraction(2) ** e2 > value:
        e2 -= 1
    mant = int(value / Fraction(2) ** (e2 - 7)) - 128
    return sign | ((e2 + 127) << 7) | mant


def unpack_codes(Wp: np.ndarray) -> np.ndarray:
    """[N, K/2] packed bytes -> [N, K] codes 0..15 (code 2j in the low nibble)."""
    lo, hi = Wp & 15, Wp >> 4
    return np.stack([lo, hi], axis=-1).reshape(Wp.shape[0], -1).astype(np.int64)


def check_route(xb, Wp, s16, o16, bias):
    M, K = xb.shape
    N, G = s16.shape
    q = unpack_codes(Wp)
    y_o, xq, sx, xsum, acc = oracle.w4a8_linear(xb, Wp, s16, o16, bias)
    xq = xq.astype(np.int64)
    exact_matches = 0
    planes_needed = 0
    for n in range(N):
        s = [f16_value(int(b)) for b in s16[n]]
        o = [f16_value(int(b)) for b in o16[n]]
        nz = [v for v in s + o if v != 0]
        e_n = min(lowest_bit_exponent(v) for v in nz) if nz else 0
        S = [v / Fraction(2) ** e_n for v in s]
        O = [v / Fraction(2) ** e_n for v in o]
        assert all(v.denominator == 1 for v in S + O)  # the integer grid
        S = np.array([int(v) for v in S], dtype=object)
        O = np.array([int(v) for v in O], dtype=object)
        W = S[np.arange(K) // 64] * q[n].astype(object) + O[np.arange(K) // 64]
        # every dequantized weight is 2^e_n W
        for k in range(0, K, 37):
            assert Fraction(int(W[k])) * Fraction(2) ** e_n == s[k // 64] * int(q[n, k]) + o[k // 64]
        # the signed digits of the fewest bytes that hold U = W + 0x80..80
        P = 1
        while not all(0 <= int(w) + sum(128 * 256 ** p for p in range(P)) < 256 ** P for w in W):
            P += 1
        planes_needed = max(planes_needed, P)
        c = sum(128 * 256 ** p for p in range(P))
        U = [int(w) + c for w in W]
        digits = [[((u >> (8 * p)) & 255) - 128 for u in U] for p in range(P)]
        assert all(-128 <= d <= 127 for dp in digits for d in dp)
        assert all(sum(256 ** p * digits[p][k] for p in range(P)) == int(W[k]) for k in range(K))
        for m in range(M):
            # P digit GEMMs, weighted by 256^p, give the integer GEMM ...
            Yp = [sum(int(xq[m, k]) * digits[p][k] for k in range(K)) for p in range(P)]
            Y = sum(256 ** p * Yp[p] for p in range(P))
            assert Y == sum(int(xq[m, k]) * int(W[k]) for k in range(K))
            # ... and 2^e_n Y is the per-group fold, exactly
            fold = sum(s[g] * int(acc[m, n, g]) + o[g] * int(xsum[m, g]) for g in range(G))
            assert Fraction(Y) * Fraction(2) ** e_n == fold
            # the route's single rounding against the oracle's output
            v = Fraction(float(sx[m])) * Fraction(2) ** e_n * Y
            if bias is not None:
                v += Fraction(float(bias[n]))
            want = bf16_rne(v)
            d = bf16_ulp_distance(np.array([want], np.uint16), y_o[m:m + 1, n])
            assert d.max() <= 1, (m, n)
            exact_matches += int(want == int(y_o[m, n]))
    return exact_matches, planes_needed


def test_gaussian_weights():
    case = synthetic.LinearCase("pl", M=3, K=256, N=16, bias=True, outlier_frac=0.01, seed=7)
    xb, W, b, _ = case.draw()
    Wp, s16, o16 = oracle.quant_w4(W)
    exact, P = check_route(xb, Wp, s16, o16, b)
    assert P in (2, 3)
    assert exact >= 3 * 16 - 1  # the fold is exact in fp64 on these sizes


def test_integer_groups_and_a_subnormal_group():
    rng = np.random.default_rng(8)
    N, K = 16, 256
    G = K // 64
    Wp = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    xb = synthetic.f32_to_bf16_bits(rng.standard_normal((2, K)).astype(np.float32))
    # s = 1 and a small integer offset: one digit
    s = np.ones((N, G), np.float32)
    o = rng.integers(-8, 1, (N, G)).astype(np.float32)
    s16 = s.astype(np.float16).view(np.uint16)
    o16 = o.astype(np.float16).view(np.uint16)
    exact, P = check_route(xb, Wp, s16, o16, None)
    assert P == 1 and exact == 2 * N
    # typical scales with one subnormal group per row: the grid moves to 2^-24
    s = rng.uniform(0.004, 0.009, (N, G)).astype(np.float32)
    o = -rng.uniform(0.02, 0.06, (N, G)).astype(np.float32)
    s[:, 1] = 3e-6
    o[:, 1] = -2e-5
    s16 = s.astype(np.float16).view(np.uint16)
    o16 = o.astype(np.float16).view(np.uint16)
    exact, P = check_route(xb, Wp, s16, o16, None)
    assert P == 3


def test_the_rounding_helper_matches_the_oracle():
    rng = np.random.default_rng(9)
    for v in rng.standard_normal(300) * np.exp(rng.uniform(-30, 30, 300)):
        assert bf16_rne(Fraction(float(v))) == oracle.f64_to_bf16(float(v))
    assert bf16_rne(Fraction(1) + Fraction(1, 256)) == 0x3F80        # a tie, to even
    assert bf16_rne(Fraction(1) + Fraction(3, 256)) == 0x3F82
    assert bf16_rne(Fraction(2) - Fraction(1, 512)) == 0x4000        # carry into the next binade
