"""Pins for the CPU oracle, checked against things other than itself.

Each test pins one part of the oracle to a closed form, an invariant that the
definitions fix, an independent library routine (numpy / torch CPU), a
hand-derived fixture under ``tests/golden/``, or brute force on tiny inputs.
They are chosen so that a plausible slip in the oracle (a dropped term, a wrong
sign or index, a transposed operand, the wrong rounding rule) fails one of them.
No GPU is needed.
"""
import json
import math
import os

import numpy as np
import pytest

from w4a8_quantized_gemm_token_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(a):
    return synthetic.f32_to_bf16_bits(np.asarray(a, np.float32))


def bf16_val(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def ordinal(bits):
    """Map bf16 bit patterns to integers that are monotone in the value (+0 == -0)."""
    b = np.asarray(bits, np.uint16).astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


# --------------------------------------------------------------- encodings

def test_f64_to_bf16_exhaustive_neighbours(orc):
    """Every finite bf16 maps to itself; midpoints go to the even neighbour, and
    anything off the midpoint goes to the nearer one (IEEE round-to-nearest-even)."""
    f = orc._load().oracle_f64_to_bf16
    for b in range(1, 0x7F80):
        v = float(bf16_val(b))
        assert f(v) == b and f(-v) == (b | 0x8000)
        if b < 0x7F7F:
            nxt = float(bf16_val(b + 1))
            mid = (v + nxt) / 2.0          # exact in double
            even = b if b % 2 == 0 else b + 1
            assert f(mid) == even, hex(b)
            assert f(-mid) == (even | 0x8000)
            assert f(math.nextafter(mid, math.inf)) == b + 1
            assert f(math.nextafter(mid, -math.inf)) == b
    # top of the range: the midpoint to 2^128 ties to even (0x7F80 = inf)
    top = float(bf16_val(0x7F7F))
    mid = (top + 2.0 ** 128) / 2.0
    assert f(math.nextafter(mid, -math.inf)) == 0x7F7F
    assert f(mid) == 0x7F80
    assert f(1e300) == 0x7F80 and f(-1e300) == 0xFF80
    assert f(0.0) == 0 and f(-0.0) == 0x8000
    # below the smallest bf16 subnormal 2^-133: half of it ties to zero (even)
    assert f(2.0 ** -134) == 0 and f(math.nextafter(2.0 ** -134, 1.0)) == 1


def test_f16_conversions_match_numpy(orc):
    """fp32 -> fp16 rounding and fp16 -> fp32 widening agree with numpy's float16."""
    allbits = np.arange(0x10000, dtype=np.uint16)
    finite = allbits[np.isfinite(allbits.view(np.float16))]
    f16_to_f32 = orc._load().oracle_f16_to_f32
    got = np.array([f16_to_f32(int(u)) for u in finite], np.float32)
    assert np.array_equal(got, finite.view(np.float16).astype(np.float32))

    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * 0.02,
        rng.standard_normal(2000).astype(np.float32) * 100,
        # exact fp16 midpoints (ties) in several binades
        (finite.view(np.float16).astype(np.float32)[1000:3000:7] * np.float32(1 + 2 ** -11)),
    ]).astype(np.float32)
    to16 = orc._load().oracle_f32_to_f16
    got = np.array([to16(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, vals.astype(np.float16).view(np.uint16))


# ------------------------------------------------------- activation quant

def test_quant_golden_rows(orc):
    """Hand-derived rows (exact ties, power-of-two scales, the zero row)."""
    with open(os.path.join(GOLDEN, "quant_act_rows.json")) as fh:
        fx = json.load(fh)
    for row in fx["rows"]:
        x = bf16_bits([row["x"]])
        assert np.array_equal(bf16_val(x)[0], np.float32(row["x"]))  # inputs exact in bf16
        xq, sx = orc.quant_act(x)
        assert xq[0].tolist() == row["codes"]
        assert float(sx[0]) == row["scale"]


def test_quant_integer_rows_closed_form(orc):
    """Integer rows whose absmax is 127 quantize to themselves with scale 1."""
    rng = np.random.default_rng(2)
    x = rng.integers(-127, 128, size=(33, 96)).astype(np.float32)
    x[np.arange(33), rng.integers(0, 96, 33)] = np.where(rng.random(33) < 0.5, 127, -127)
    xq, sx = orc.quant_act(bf16_bits(x))
    assert np.array_equal(xq.astype(np.float32), x)
    assert np.all(sx == 1.0)


def test_quant_single_nonzero_and_zero(orc):
    x = np.zeros((3, 64), np.float32)
    x[1, 5] = -3.0
    x[2, 63] = 1e-20
    xq, sx = orc.quant_act(bf16_bits(x))
    assert sx[0] == 1.0 and not xq[0].any()
    assert xq[1, 5] == -127 and np.count_nonzero(xq[1]) == 1
    assert sx[1] == np.float32(3.0) / np.float32(127.0)
    assert xq[2, 63] == 127 and np.count_nonzero(xq[2]) == 1


@pytest.mark.parametrize("K", [32, 96, 256, 3072])
def test_quant_error_bound_and_range(orc, K):
    """|x - q*sx| <= sx*(1/2 + 2^-15), codes in [-127, 127], absmax -> +-127, and
    sx*127 equals absmax to fp32 rounding."""
    case = synthetic.LinearCase("pin", M=40, K=K, N=8, outlier_frac=0.02, seed=K)
    xb, _, _, _ = case.draw()
    x = bf16_val(xb).astype(np.float64)
    xq, sx = orc.quant_act(xb)
    assert xq.min() >= -127 and xq.max() <= 127
    err = np.abs(x - xq.astype(np.float64) * sx[:, None].astype(np.float64))
    assert np.all(err <= sx[:, None] * (0.5 + 2.0 ** -15))
    amax = np.abs(x).max(axis=1)
    arg = np.abs(x).argmax(axis=1)
    assert np.all(np.abs(xq[np.arange(40), arg]) == 127)
    assert np.all(np.abs(sx.astype(np.float64) * 127 - amax) <= amax * 2.0 ** -23)


def test_quant_power_of_two_and_sign_invariance(orc):
    """Scaling a row by 2^j scales sx by 2^j and leaves the codes; negating the
    row negates the codes."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((16, 128)).astype(np.float32)
    xb = bf16_bits(x)
    xv = bf16_val(xb)
    xq, sx = orc.quant_act(xb)
    for j in (-3, 5):
        xq2, sx2 = orc.quant_act(bf16_bits(xv * np.float32(2.0 ** j)))
        assert np.array_equal(xq2, xq)
        assert np.array_equal(sx2, sx * np.float32(2.0 ** j))
    xq3, sx3 = orc.quant_act(bf16_bits(-xv))
    assert np.array_equal(xq3, -xq) and np.array_equal(sx3, sx)


def test_quant_ties_round_to_even_with_unit_scale(orc):
    """With absmax 127 the multiplier is exactly 1, so codes are numpy's rint."""
    rng = np.random.default_rng(4)
    halves = (rng.integers(-253, 254, size=(8, 63)) / 2.0).astype(np.float32)
    x = np.concatenate([np.full((8, 1), 127, np.float32), halves], axis=1)
    xq, sx = orc.quant_act(bf16_bits(x))
    assert np.all(sx == 1.0)
    assert np.array_equal(xq.astype(np.float32), np.rint(bf16_val(bf16_bits(x))))


def test_weight_quant_w8_bound(orc):
    """The W8 per-output-channel quant obeys the same bound on fp32 rows."""
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((24, 320)) * 0.02).astype(np.float32)
    W[3] = 0
    Wq, sw = orc.quant_w8(W)
    assert sw[3] == 1.0 and not Wq[3].any()
    err = np.abs(W.astype(np.float64) - Wq * sw[:, None].astype(np.float64))
    assert np.all(err <= sw[:, None] * (0.5 + 2.0 ** -15))
    assert np.all(np.abs(Wq).max(axis=1)[np.arange(24) != 3] == 127)


def test_group_sums_match_numpy(orc):
    rng = np.random.default_rng(6)
    xq = rng.integers(-127, 128, size=(7, 256)).astype(np.int8)
    want = xq.astype(np.int64).reshape(7, 4, 64).sum(axis=2)
    assert np.array_equal(orc.group_sums(xq), want)


# --------------------------------------------------------------------- W4

def unpack_codes(Wp):
    lo = Wp & 0x0F
    hi = Wp >> 4
    return np.stack([lo, hi], axis=-1).reshape(Wp.shape[0], -1)


def w4_golden_groups():
    """The hand-derived W4 groups of ``tests/golden/w4_affine_groups.json`` as
    (64 fp32 inputs, scale fp16 bits, offset fp16 bits, codes): the fp16 affine
    grids, and the groups given by their inputs that tell the reading R5 (codes
    from the fp16-rounded scale and offset, times the reciprocal of the scale)
    from the alternatives."""
    with open(os.path.join(GOLDEN, "w4_affine_groups.json")) as fh:
        fx = json.load(fh)
    out = []
    for grp in fx["groups"]:
        codes = np.array(grp["codes"], np.float32)
        w = np.float32(grp["offset"]) + codes * np.float32(grp["scale"])
        out.append((w, int(grp["scale_f16"], 16), int(grp["offset_f16"], 16), grp["codes"]))
    for grp in fx["groups_w"]:
        w = np.array(grp["w"], np.float32)
        assert np.array_equal(w.astype(np.float64), np.array(grp["w"], np.float64))  # exact in fp32
        out.append((w, int(grp["scale_f16"], 16), int(grp["offset_f16"], 16), grp["codes"]))
    return out


def test_w4_affine_grid_golden(orc):
    """Groups built on an fp16 affine grid come back with the same s, o and
    codes; the groups built to separate R5 from its alternatives (division by
    the scale, codes from the unrounded scale or offset) give R5's codes."""
    groups = w4_golden_groups()
    W = np.concatenate([g[0] for g in groups])[None, :]    # one row, one group each
    Wp, s, o = orc.quant_w4(W)
    for g, (_, s16, o16, codes) in enumerate(groups):
        assert s[0, g] == s16
        assert o[0, g] == o16
        assert unpack_codes(Wp)[0, 64 * g:64 * g + 64].tolist() == codes


def test_w4_pack_nibble_order(orc):
    """Code k = 2j sits in the low nibble of byte j, k = 2j + 1 in the high one."""
    codes = np.tile(np.arange(16, dtype=np.float32), 4)          # 0..15 repeated
    W = (np.float32(-1.0) + codes * np.float32(0.125))[None, :]
    Wp, s, o = orc.quant_w4(W)
    assert Wp[0, 0] == 0x10 and Wp[0, 1] == 0x32 and Wp[0, 7] == 0xFE


def test_w4_error_bound_and_degenerate(orc):
    """|w - (q*s + o)| <= s/2 + 15*|s - (hi-lo)/15| + |o - lo| (+ fp32 slack);
    a constant group gets s = 0 and zero codes."""
    rng = np.random.default_rng(7)
    W = (rng.standard_normal((12, 256)) * 0.02).astype(np.float32)
    W[5, 64:128] = np.float32(0.0123)
    Wp, s16, o16 = orc.quant_w4(W)
    q = unpack_codes(Wp).astype(np.float64).reshape(12, 4, 64)
    s = s16.view(np.float16).astype(np.float64)[:, :, None]
    o = o16.view(np.float16).astype(np.float64)[:, :, None]
    Wg = W.astype(np.float64).reshape(12, 4, 64)
    lo = Wg.min(axis=2, keepdims=True)
    hi = Wg.max(axis=2, keepdims=True)
    bound = s / 2 + 15 * np.abs(s - (hi - lo) / 15) + np.abs(o - lo) + 1e-6 * (np.abs(Wg) + s)
    assert np.all(np.abs(Wg - (q * s + o)) <= bound)
    assert q.min() >= 0 and q.max() <= 15
    assert s16[5, 1] == 0 and not q[5, 1].any()
    assert o16[5, 1] == np.float16(0.0123).view(np.uint16)


# ------------------------------------------------------------- accumulate

def test_w8a8_acc_matches_int64_matmul(orc):
    rng = np.random.default_rng(8)
    xq = rng.integers(-127, 128, size=(19, 160)).astype(np.int8)
    Wq = rng.integers(-127, 128, size=(23, 160)).astype(np.int8)
    want = xq.astype(np.int64) @ Wq.astype(np.int64).T
    assert np.array_equal(orc.w8a8_acc(xq, Wq), want)


def test_w4a8_group_acc_matches_int64(orc):
    rng = np.random.default_rng(9)
    xq = rng.integers(-127, 128, size=(5, 192)).astype(np.int8)
    Wp = rng.integers(0, 256, size=(6, 96)).astype(np.uint8)
    q = unpack_codes(Wp).astype(np.int64)
    want = np.einsum("mgk,ngk->mng", xq.astype(np.int64).reshape(5, 3, 64), q.reshape(6, 3, 64))
    assert np.array_equal(orc.w4a8_group_acc(xq, Wp), want)
    # one-hot activations read back single codes: the unpack is the pack's inverse
    eye = np.zeros((192, 192), np.int8)
    eye[np.arange(192), np.arange(192)] = 1
    acc = orc.w4a8_group_acc(eye, Wp)          # [192, N, 3]
    codes_back = acc[np.arange(192), :, np.arange(192) // 64].T
    assert np.array_equal(codes_back, q)


# ------------------------------------------------------------ whole linear

def test_w8a8_integer_closed_form(orc):
    """Integer x and W with row absmax 127 give sx = sw = 1, xq = x, Wq = W, and
    y = bf16(x @ W^T + bias) exactly (torch's fp32 -> bf16 rounding is exact here
    because the sums are integers below 2^24)."""
    import torch

    rng = np.random.default_rng(10)
    M, K, N = 17, 64, 24
    x = rng.integers(-127, 128, size=(M, K)).astype(np.float32)
    x[:, 0] = 127
    W = rng.integers(-127, 128, size=(N, K)).astype(np.float32)
    W[:, 1] = -127
    bias = rng.integers(-1000, 1000, size=N).astype(np.float32)
    Wq, sw = orc.quant_w8(W)
    assert np.all(sw == 1.0) and np.array_equal(Wq.astype(np.float32), W)
    y, xq, sx, acc = orc.w8a8_linear(bf16_bits(x), Wq, sw, bias)
    exact = x.astype(np.int64) @ W.astype(np.int64).T
    assert np.array_equal(acc, exact)
    ref = torch.from_numpy((exact + bias.astype(np.int64)).astype(np.float32))
    want = ref.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(y, want)
    y0, _, _, _ = orc.w8a8_linear(bf16_bits(x), Wq, sw, None)
    want0 = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(y0, want0.view(torch.int16).numpy().view(np.uint16))


def test_w8a8_dequant_brute_force(orc):
    """The factored dequant equals sum_k (xq*sx)(wq*sw) + bias term by term in fp64."""
    case = synthetic.LinearCase("pin", M=9, K=96, N=11, outlier_frac=0.03, seed=11)
    xb, W, b, _ = case.draw()
    Wq, sw = orc.quant_w8(W)
    xq, sx = orc.quant_act(xb)
    acc = orc.w8a8_acc(xq, Wq)
    v = orc.w8a8_dequant_f64(acc, sx, sw, b)
    xd = xq.astype(np.float64) * sx.astype(np.float64)[:, None]
    wd = Wq.astype(np.float64) * sw.astype(np.float64)[:, None]
    terms = xd[:, None, :] * wd[None, :, :]
    brute = terms.sum(axis=2) + b.astype(np.float64)
    scale = np.abs(terms).sum(axis=2) + np.abs(b)
    assert np.all(np.abs(v - brute) <= 1e-12 * scale)
    y = orc.w8a8_dequant(acc, sx, sw, b)
    assert np.array_equal(y, orc.f64_to_bf16_array(v))


def test_w8a8_within_quantization_bound_of_exact(orc):
    """y lies within sum_k(|x|e_w + |w|e_x + e_x e_w) (+ bf16 rounding) of the
    unquantized fp64 x . W^T + bias; a transposed or mis-scaled operand would not."""
    case = synthetic.LinearCase("pin", M=12, K=128, N=20, outlier_frac=0.02, seed=12)
    xb, W, b, _ = case.draw()
    Wq, sw = orc.quant_w8(W)
    y, xq, sx, _ = orc.w8a8_linear(xb, Wq, sw, b)
    x = bf16_val(xb).astype(np.float64)
    Wd = W.astype(np.float64)
    exact = x @ Wd.T + b
    ex = (sx.astype(np.float64) * (0.5 + 2.0 ** -15))[:, None]
    ew = (sw.astype(np.float64) * (0.5 + 2.0 ** -15))[:, None]
    bound = (np.abs(x).sum(axis=1)[:, None] * ew.T
             + ex * np.abs(Wd).sum(axis=1)[None, :]
             + ex * ew.T * 128)
    yv = bf16_val(y).astype(np.float64)
    assert np.all(np.abs(yv - exact) <= bound + np.abs(yv) * 2.0 ** -8 + 1e-30)
    # quantization noise is a few percent of the output (a dropped bias, a wrong
    # scale or a transposed operand would be of the output's own size)
    rms = lambda a: float(np.sqrt(np.mean(a * a)))
    assert rms(yv - exact) < 0.05 * rms(exact)


def test_w4a8_dequant_brute_force(orc):
    """sx * sum_g(s acc_g + o xsum_g) + bias equals sum_k (xq*sx)*(q*s + o) + bias."""
    case = synthetic.LinearCase("pin", M=6, K=256, N=10, seed=13)
    xb, W, b, _ = case.draw()
    Wp, s16, o16 = orc.quant_w4(W)
    xq, sx = orc.quant_act(xb)
    xsum = orc.group_sums(xq)
    acc = orc.w4a8_group_acc(xq, Wp)
    v = orc.w4a8_dequant_f64(acc, xsum, sx, s16, o16, b)
    q = unpack_codes(Wp).astype(np.float64)
    s = np.repeat(s16.view(np.float16).astype(np.float64), 64, axis=1)
    o = np.repeat(o16.view(np.float16).astype(np.float64), 64, axis=1)
    wd = q * s + o
    xd = xq.astype(np.float64) * sx.astype(np.float64)[:, None]
    terms = xd[:, None, :] * wd[None, :, :]
    brute = terms.sum(axis=2) + b
    scale = np.abs(terms).sum(axis=2) + np.abs(b)
    assert np.all(np.abs(v - brute) <= 1e-12 * scale)
    y = orc.w4a8_dequant(acc, xsum, sx, s16, o16, b)
    assert np.array_equal(y, orc.f64_to_bf16_array(v))
    # no-bias form (the W4A8 workload has none)
    v0 = orc.w4a8_dequant_f64(acc, xsum, sx, s16, o16, None)
    assert np.all(np.abs(v0 - (brute - b)) <= 1e-12 * scale)


def test_w4a8_within_quantization_bound_of_exact(orc):
    case = synthetic.LinearCase("pin", M=8, K=192, N=12, seed=14, bias=False)
    xb, W, _, _ = case.draw()
    Wp, s16, o16 = orc.quant_w4(W)
    y, xq, sx, xsum, acc = orc.w4a8_linear(xb, Wp, s16, o16, None)
    x = bf16_val(xb).astype(np.float64)
    Wd = W.astype(np.float64)
    exact = x @ Wd.T
    q = unpack_codes(Wp).astype(np.float64)
    s = np.repeat(s16.view(np.float16).astype(np.float64), 64, axis=1)
    o = np.repeat(o16.view(np.float16).astype(np.float64), 64, axis=1)
    ew = np.abs(Wd - (q * s + o))                    # per-weight error (bounded above)
    ex = (sx.astype(np.float64) * (0.5 + 2.0 ** -15))[:, None]
    bound = np.abs(x) @ ew.T + ex * np.abs(Wd).sum(axis=1)[None, :] + ex @ ew.sum(axis=1)[None, :]
    yv = bf16_val(y).astype(np.float64)
    assert np.all(np.abs(yv - exact) <= bound + np.abs(yv) * 2.0 ** -8 + 1e-30)
    rms = lambda a: float(np.sqrt(np.mean(a * a)))
    assert rms(yv - exact) < 0.1 * rms(exact)


# ----------------------------------------------- gated residual epilogue

def test_w8a8_gated_integer_closed_form(orc):
    """Integer x and W with row absmax 127 (sx = sw = 1), an integer bias and
    residual and power-of-two gates: out = bf16(r + g * (x @ W^T + bias)),
    computed here in numpy int64 / float32 (exact: every value is a multiple of
    1/4 below 2^22) and rounded by torch."""
    import torch

    rng = np.random.default_rng(12)
    M, K, N = 13, 64, 24
    x = rng.integers(-127, 128, size=(M, K)).astype(np.float32)
    x[:, 3] = -127
    W = rng.integers(-127, 128, size=(N, K)).astype(np.float32)
    W[:, 5] = 127
    bias = rng.integers(-1000, 1000, size=N).astype(np.float32)
    gate = rng.choice(np.array([0.25, -0.5, 1.0, 2.0, -4.0], np.float32), size=N)
    r = rng.integers(-200, 200, size=(M, N)).astype(np.float32)  # exact in bf16
    Wq, sw = orc.quant_w8(W)
    out, xq, sx, acc = orc.w8a8_linear_gated(bf16_bits(x), Wq, sw, bias, gate, bf16_bits(r))
    exact = x.astype(np.int64) @ W.astype(np.int64).T + bias.astype(np.int64)
    want_f = (r.astype(np.float64) + gate.astype(np.float64) * exact).astype(np.float32)
    want = torch.from_numpy(want_f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(out, want)


def test_w8a8_gated_zero_gate_and_unit_gate(orc):
    """A zero gate returns the residual bit for bit; a unit gate with a zero
    residual returns the plain linear (whose own pins are above)."""
    case = synthetic.LinearCase("gz", M=7, K=160, N=16, outlier_frac=0.05, seed=13)
    xb, W, b, _ = case.draw()
    Wq, sw = orc.quant_w8(W)
    rng = np.random.default_rng(14)
    r = bf16_bits(rng.normal(size=(7, 16)).astype(np.float32) * 3)
    out0, _, _, _ = orc.w8a8_linear_gated(xb, Wq, sw, b, np.zeros(16, np.float32), r)
    assert np.array_equal(out0, r)
    out1, _, _, _ = orc.w8a8_linear_gated(xb, Wq, sw, b, np.ones(16, np.float32),
                                          np.zeros((7, 16), np.uint16))
    y, _, _, _ = orc.w8a8_linear(xb, Wq, sw, b)
    assert np.array_equal(out1, y)


def test_w8a8_gated_brute_force(orc):
    """r + g * (sum_k (xq*sx)(wq*sw) + bias), term by term in fp64 and rounded by
    the (separately pinned) fp64 -> bf16 rounding, agrees with the oracle to
    within one bf16 ulp (equal unless the two fp64 evaluation orders straddle a
    rounding boundary)."""
    case = synthetic.LinearCase("gb", M=9, K=96, N=11, outlier_frac=0.03, seed=15)
    xb, W, b, _ = case.draw()
    Wq, sw = orc.quant_w8(W)
    rng = np.random.default_rng(16)
    gate = (rng.normal(size=11) * 0.5).astype(np.float32)
    r = bf16_bits(rng.normal(size=(9, 11)).astype(np.float32))
    out, xq, sx, _ = orc.w8a8_linear_gated(xb, Wq, sw, b, gate, r)
    xd = xq.astype(np.float64) * sx.astype(np.float64)[:, None]
    wd = Wq.astype(np.float64) * sw.astype(np.float64)[:, None]
    lin = (xd[:, None, :] * wd[None, :, :]).sum(axis=2) + b.astype(np.float64)
    brute = bf16_val(r).astype(np.float64) + gate.astype(np.float64) * lin
    want = orc.f64_to_bf16_array(brute)
    assert np.abs(ordinal(out) - ordinal(want)).max() <= 1
    assert np.mean(out == want) > 0.95


# ------------------------------------------------- INT8 attention (R14)

def _qkv(L, D, seed, scale_q=1.0):
    rng = np.random.default_rng(seed)
    q = bf16_bits(rng.normal(size=(L, D)) * scale_q)
    k = bf16_bits(rng.normal(size=(L, D)))
    v = bf16_bits(rng.normal(size=(L, D)))
    return q, k, v


def test_sage_single_key_returns_its_value(orc):
    """One key: its softmax weight is 1, so the output is that value row."""
    q, k, v = _qkv(1, 128, 21)
    assert np.array_equal(orc.sage_attention_head(q, k, v, 128 ** -0.5), v)


def test_sage_zero_scale_averages_the_values(orc):
    """scale = 0 makes every score 0: uniform weights, the output is the mean of
    the value rows (closed form), whatever q and k are."""
    q, k, v = _qkv(37, 128, 22)
    out = orc.sage_attention_head(q, k, v, 0.0)
    want = orc.f64_to_bf16_array(bf16_val(v).astype(np.float64).mean(axis=0))
    assert np.abs(ordinal(out) - ordinal(np.broadcast_to(want, out.shape))).max() <= 1
    assert np.mean(out == want[None, :]) > 0.95


def test_sage_key_permutation_invariance(orc):
    """Permuting the keys together with their values leaves every output."""
    q, k, v = _qkv(48, 128, 23)
    perm = np.random.default_rng(24).permutation(48)
    o1, f1 = orc.sage_attention_head(q, k, v, 128 ** -0.5, with_f64=True)
    o2, f2 = orc.sage_attention_head(q, k[perm], v[perm], 128 ** -0.5, with_f64=True)
    assert np.allclose(f1, f2, rtol=1e-12, atol=1e-15)
    assert np.abs(ordinal(o1) - ordinal(o2)).max() <= 1


def test_sage_dominant_key_selects_its_value(orc):
    """A key aligned with query 0 and far larger than the others takes all of
    query 0's weight (the next weight is below exp(-60))."""
    q, k, v = _qkv(16, 128, 25)
    k = k.copy()
    k[5] = bf16_bits(bf16_val(q[0]) * 64.0)
    others = np.delete(np.arange(16), 5)
    k[others] = bf16_bits(bf16_val(k[others]) * 0.01)
    out = orc.sage_attention_head(q, k, v, 1.0)
    assert np.array_equal(out[0], v[5])


def test_sage_close_to_unquantized_attention(orc):
    """The pages quote ~1 % total quantization error against fp32 attention;
    with Gaussian q, k, v (head dim 128, 256 tokens) the INT8 scores keep the
    output within 5 % (relative, max over elements) of fp64 attention on the
    unquantized inputs, and far from attention with the keys shuffled."""
    L, D = 256, 128
    q, k, v = _qkv(L, D, 26, scale_q=2.0)
    _, o64 = orc.sage_attention_head(q, k, v, D ** -0.5, with_f64=True)
    qf, kf, vf = (bf16_val(t).astype(np.float64) for t in (q, k, v))
    s = qf @ kf.T * D ** -0.5
    p = np.exp(s - s.max(axis=1, keepdims=True))
    ref = (p @ vf) / p.sum(axis=1, keepdims=True)
    err = np.abs(o64 - ref).max() / np.abs(ref).max()
    assert err < 0.05
    perm = np.random.default_rng(27).permutation(L)
    s2 = qf @ kf[perm].T * D ** -0.5
    p2 = np.exp(s2 - s2.max(axis=1, keepdims=True))
    wrong = (p2 @ vf) / p2.sum(axis=1, keepdims=True)
    assert np.abs(o64 - wrong).max() / np.abs(ref).max() > 10 * err


# ------------------------------------------------------------ threading

def test_thread_count_does_not_change_results(orc):
    """The row loops may run on several OpenMP threads (the CPU baseline's
    multi-core leg); every output is still computed by one thread in the same
    order, so 1 and 4 threads give the same bits."""
    case = synthetic.LinearCase("thr", M=37, K=256, N=40, outlier_frac=0.02, seed=31)
    xb, W, b, _ = case.draw()
    outs = []
    try:
        for n in (1, 4):
            orc.set_threads(n)
            Wq, sw = orc.quant_w8(W)
            Wp, s16, o16 = orc.quant_w4(W)
            y8 = orc.w8a8_linear(xb, Wq, sw, b)
            y4 = orc.w4a8_linear(xb, Wp, s16, o16, b)
            q, k, v = (xb[:32, :128], xb[1:33, :128], xb[2:34, :128])
            att = orc.sage_attention_head(q, k, v, 128 ** -0.5)
            outs.append([Wq, sw, Wp, s16, o16, *y8, *y4, att])
    finally:
        orc.set_threads(1)
    for a, c in zip(*outs):
        assert np.array_equal(a, c)
