"""The W4A8 GEMM route (M > 16) on the GPU: the byte-plane GEMM and its fallback.

The route first counts the byte planes a weight needs: with e_n the smallest
exponent of the lowest set bit over the nonzero fp16 scales and offsets of
weight row n, every dequantized weight s q + o of the row is 2^e_n times the
integer S q + O; P is the fewest bytes holding S q + O + 0x80..80 for every
code of every row (1..3), else the per-group fold kernel computes the product.

Each test builds weights of a known plane count (scales and offsets written
directly as fp16, or through the quantizer), checks the device's count against
a count written here from the fp16 bits, and the outputs against the oracle
within 2 bf16 ulp.  The planes compute the exact value of the fold, and on
these shapes the per-group fp64 fold is exact too, so the GEMM route must also
equal, bit for bit, the per-group fold kernel (QK_ROUTE_GEMM_FOLD)."""
import numpy as np
import pytest
import torch

from tests.gpu_common import host, qk, t2bits, to_dev, to_dev_bf16  # noqa: F401
from tests.helpers import bf16_ulp_distance
from w4a8_quantized_gemm_token_b200 import synthetic

pytestmark = pytest.mark.gpu

TOL_ULP = 2
GEMM, FOLD = 1, 3


def host_row_planes(s16, o16):
    """Digits each weight row needs (1..3, or 255), from the fp16 bits (numpy,
    int64; a shift past 40 bits or a non-finite value gives 255)."""
    out = []
    for n in range(np.asarray(s16).shape[0]):
        out.append(host_plane_count(np.asarray(s16)[n:n + 1], np.asarray(o16)[n:n + 1], 0))
    return np.array(out)


def host_mixed(s16, o16, K):
    """Whether a three-digit weight takes the mixed layout: at most 8 rows
    needing a third digit in every aligned block of 60 rows."""
    if host_plane_count(s16, o16, K) != 3:
        return False
    wide = host_row_planes(s16, o16) == 3
    n = len(wide)
    return all(wide[b:b + 60].sum() <= 8 for b in range(0, n, 60))


def host_plane_count(s16, o16, K):
    """The plane count from the fp16 bits (numpy, int64; a shift past 40 bits
    or a non-finite value gives 255)."""
    bits = np.stack([np.asarray(s16, np.uint16), np.asarray(o16, np.uint16)]).astype(np.int64)
    E = (bits >> 10) & 31
    m = bits & 1023
    mant = np.where(E != 0, m | 1024, m)
    L = np.where(E != 0, E - 25, -24)
    if (E == 31).any():
        return 255
    tz = np.zeros_like(mant)
    v = mant.copy()
    for _ in range(11):
        z = (v != 0) & ((v & 1) == 0)
        tz += z
        v = np.where(z, v >> 1, v)
    low = np.where(mant != 0, L + tz, 1 << 20)
    eb = low.min(axis=(0, 2))                       # per weight row
    eb = np.where(eb == 1 << 20, 0, eb)[None, :, None]
    sh = L - eb
    if ((mant != 0) & (sh > 40)).any():
        return 255
    val = np.where(sh >= 0, mant << np.maximum(sh, 0), mant >> np.maximum(-sh, 0))
    val = np.where(bits & 0x8000, -val, val)
    S, O = val[0], val[1]
    lo = np.minimum(O, O + 15 * S).min()
    hi = np.maximum(O, O + 15 * S).max()
    for p in range(1, 4):
        c = sum(0x80 << (8 * i) for i in range(p))
        if lo + c >= 0 and hi + c < (1 << (8 * p)):
            return p
    return 255


def fp16_bits(a):
    return np.asarray(a, np.float32).astype(np.float16).view(np.uint16)


def make_weights(orc, kind, N, K, seed):
    """(Wp uint8 [N, K/2], s16, o16 fp16 bits [N, K/64], the plane counts the
    construction allows: Gaussian weights need 2, a few rows 3; a tiny group
    needs K >= 128 to have a partner group)."""
    rng = np.random.default_rng(seed)
    G = K // 64
    if kind == "gauss":
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        Wp, s16, o16 = orc.quant_w4(W)
        return Wp, s16, o16, (2, 3)
    Wp = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    if kind == "unit":
        # s = 1, o a small integer: S q + O = q + o in [-8, 15], one byte
        s = np.ones((N, G), np.float32)
        o = rng.integers(-8, 1, (N, G)).astype(np.float32)
        return Wp, fp16_bits(s), fp16_bits(o), (1,)
    # scales and offsets of a typical range, then per row one group far below
    # it (subnormal fp16, lowest bit 2^-24) that moves the grid down
    base = {"p3": (0.004, 0.009, 0.02, 0.06), "p4": (0.5, 1.0, 2.0, 8.0),
            "fold": (10.0, 40.0, 100.0, 400.0), "negscale": (0.004, 0.009, 0.02, 0.06)}[kind]
    s = rng.uniform(base[0], base[1], (N, G)).astype(np.float32)
    o = -rng.uniform(base[2], base[3], (N, G)).astype(np.float32)
    if kind == "negscale":
        # a negative scale with the offset at the group maximum: the same
        # weights read downwards (the format allows it; the quantizer never
        # writes it); no tiny group, so two planes
        neg = rng.random((N, G)) < 0.3
        o = np.where(neg, o + 15 * s, o)
        s = np.where(neg, -s, s)
        return Wp, fp16_bits(s), fp16_bits(o), (2, 3)
    g0 = rng.integers(0, G, N)
    s[np.arange(N), g0] = rng.uniform(1e-6, 5e-6, N)
    o[np.arange(N), g0] = -rng.uniform(1e-5, 3e-5, N)
    # four bytes are beyond the plane GEMM: those weights take the fold
    allowed = {"p3": (3,), "p4": (255,), "fold": (255,)}[kind] if G > 1 else (2, 3)
    return Wp, fp16_bits(s), fp16_bits(o), allowed


def dev_fp16(bits):
    return to_dev(np.ascontiguousarray(bits, np.uint16).view(np.float16))


def run_both_routes(qk, orc, xb, Wp, s16, o16, b, M, K, N):
    x = to_dev_bf16(xb)
    dw = (to_dev(Wp), dev_fp16(s16), dev_fp16(o16))
    bias = to_dev(b) if b is not None else None
    xq, sx, xsum = qk.qk_quantize_activations(x, with_xsum=True)
    y_g = qk.qk_w4a8_gemm(xq, sx, xsum, *dw, bias, route=GEMM)
    y_f = qk.qk_w4a8_gemm(xq, sx, xsum, *dw, bias, route=FOLD)
    torch.cuda.synchronize()
    y_o, xq_o, _, _, _ = orc.w4a8_linear(xb, Wp, s16, o16, b)
    assert np.array_equal(host(xq), xq_o)
    return x, dw, bias, y_g, y_f, y_o


KINDS = ["gauss", "unit", "p3", "p4", "fold", "negscale"]


@pytest.mark.parametrize("kind", KINDS)
def test_plane_count(qk, orc, kind):
    N, K = 136, 1024
    Wp, s16, o16, allowed = make_weights(orc, kind, N, K, seed=len(kind))
    expect = host_plane_count(s16, o16, K)
    assert expect in allowed
    assert qk.qk_debug_w4a8_plane_count(dev_fp16(s16), dev_fp16(o16), K) == expect


def test_plane_count_special_rows(qk, orc):
    """All-zero rows add no constraint; an infinite scale sends the product to
    the fold."""
    N, K = 64, 1024
    Wp, s16, o16, _ = make_weights(orc, "gauss", N, K, seed=5)
    s16 = s16.copy()
    o16 = o16.copy()
    s16[3] = 0
    o16[3] = 0
    assert qk.qk_debug_w4a8_plane_count(dev_fp16(s16), dev_fp16(o16), K) == host_plane_count(s16, o16, K)
    s16[7, 2] = 0x7C00  # +inf
    assert host_plane_count(s16, o16, K) == 255
    assert qk.qk_debug_w4a8_plane_count(dev_fp16(s16), dev_fp16(o16), K) == 255


# M: one pair tile, a ragged second tile; N: less than one tile, ragged tiles
# at every plane count (tiles of 256 / 128 / 64 weight rows); K: an odd group
# count (a half-empty last K block) and several stages
SHAPES = [(17, 192, 72), (300, 1024, 264), (257, 320, 136), (512, 4096, 512), (64, 64, 8)]


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("MKN", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_gemm_route_parity(qk, orc, kind, MKN):
    M, K, N = MKN
    Wp, s16, o16, allowed = make_weights(orc, kind, N, K, seed=M + K + N)
    expect = host_plane_count(s16, o16, K)
    assert expect in allowed
    assert qk.qk_debug_w4a8_plane_count(dev_fp16(s16), dev_fp16(o16), K, with_mixed=True) == \
        (expect, host_mixed(s16, o16, K))
    case = synthetic.LinearCase("pl", M=M, K=K, N=N, bias=True, outlier_frac=0.01, seed=M * 3 + N)
    xb, _, b, _ = case.draw()
    _, _, _, y_g, y_f, y_o = run_both_routes(qk, orc, xb, Wp, s16, o16, b, M, K, N)
    d = bf16_ulp_distance(t2bits(y_g), y_o)
    assert d.max() <= TOL_ULP, f"{kind}: worst {d.max()} ulp"
    assert bf16_ulp_distance(t2bits(y_f), y_o).max() <= TOL_ULP
    assert torch.equal(y_g.view(torch.int16), y_f.view(torch.int16)), kind
    qk.qk_check_device_error()


def test_mixed_layout_boundaries(qk, orc):
    """The mixed layout at its edges: a 60-row block with exactly 8 rows needing
    a third digit (mixed) and one with 9 (uniform three planes), ragged N, and
    the rows needing it at the first and last positions of a block."""
    M, K = 300, 1024
    G = K // 64
    rng = np.random.default_rng(7)
    for N, wide_rows, mixed in [(136, [0, 7, 20, 33, 41, 50, 58, 59], True),
                                (136, [0, 7, 20, 33, 41, 50, 58, 59, 30], False),
                                (264, [60, 119, 120, 179, 263], True)]:
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        Wp, s16, o16 = orc.quant_w4(W)
        s = s16.view(np.float16).astype(np.float32)
        o = o16.view(np.float16).astype(np.float32)
        narrow = host_row_planes(s16, o16) <= 2
        # keep only rows that need two digits, then give the chosen rows one
        # group of a small range (subnormal fp16 scale and offset): a third digit
        for n in range(N):
            if not narrow[n]:
                s[n], o[n] = s[n - 1], o[n - 1]
        for n in wide_rows:
            s[n, 1], o[n, 1] = 3e-6, -2e-5
        s16, o16 = fp16_bits(s), fp16_bits(o)
        rows = host_row_planes(s16, o16)
        assert set(np.flatnonzero(rows == 3)) == set(wide_rows)
        assert host_mixed(s16, o16, K) == mixed
        assert qk.qk_debug_w4a8_plane_count(dev_fp16(s16), dev_fp16(o16), K, with_mixed=True) == (3, mixed)
        case = synthetic.LinearCase("mx", M=M, K=K, N=N, bias=True, seed=N + len(wide_rows))
        xb, _, b, _ = case.draw()
        _, _, _, y_g, y_f, y_o = run_both_routes(qk, orc, xb, Wp, s16, o16, b, M, K, N)
        assert bf16_ulp_distance(t2bits(y_g), y_o).max() <= TOL_ULP
        assert torch.equal(y_g.view(torch.int16), y_f.view(torch.int16))
    qk.qk_check_device_error()


@pytest.mark.parametrize("kind", ["gauss", "p3"])
def test_gemm_route_large_k(qk, orc, kind):
    """K = 65536 (1024 groups): the byte sums stay exact in int32 and Y in fp64."""
    M, K, N = 40, 65536, 72
    Wp, s16, o16, allowed = make_weights(orc, kind, N, K, seed=11)
    expect = host_plane_count(s16, o16, K)
    assert expect in allowed
    assert qk.qk_debug_w4a8_plane_count(dev_fp16(s16), dev_fp16(o16), K) == expect
    case = synthetic.LinearCase("lk", M=M, K=K, N=N, bias=False, seed=12)
    xb, _, _, _ = case.draw()
    _, _, _, y_g, y_f, y_o = run_both_routes(qk, orc, xb, Wp, s16, o16, None, M, K, N)
    assert bf16_ulp_distance(t2bits(y_g), y_o).max() <= TOL_ULP
    assert bf16_ulp_distance(t2bits(y_f), y_o).max() <= TOL_ULP


def test_workspace_reuse_across_plane_counts(qk, orc):
    """One workspace for calls whose weights need 2, 3, 255 (fold) and 1
    planes, first filled with garbage: the plane-count word of each call is
    tagged with that call's epoch, so a word left by an earlier call (or
    anything else) never decides a later one."""
    M, K, N = 300, 1024, 264
    case = synthetic.LinearCase("ws", M=M, K=K, N=N, bias=True, seed=21)
    xb, _, b, _ = case.draw()
    x = to_dev_bf16(xb)
    bias = to_dev(b)
    nbytes = qk.qk_w4a8_workspace_size(M, K)
    ws = torch.randint(-128, 128, (nbytes,), dtype=torch.int8, device="cuda")
    for i, kind in enumerate(["gauss", "p3", "fold", "unit", "gauss"]):
        Wp, s16, o16, _ = make_weights(orc, kind, N, K, seed=30 + i)
        y = qk.qk_w4a8_linear(x, to_dev(Wp), dev_fp16(s16), dev_fp16(o16), bias, workspace=ws)
        torch.cuda.synchronize()
        y_o, _, _, _, _ = orc.w4a8_linear(xb, Wp, s16, o16, b)
        assert bf16_ulp_distance(t2bits(y), y_o).max() <= TOL_ULP, kind
    # the word itself: 0xFF.. in every byte (an epoch this process never uses)
    ws.fill_(-1)
    Wp, s16, o16, _ = make_weights(orc, "gauss", N, K, seed=40)
    y = qk.qk_w4a8_linear(x, to_dev(Wp), dev_fp16(s16), dev_fp16(o16), bias, workspace=ws)
    torch.cuda.synchronize()
    y_o, _, _, _, _ = orc.w4a8_linear(xb, Wp, s16, o16, b)
    assert bf16_ulp_distance(t2bits(y), y_o).max() <= TOL_ULP
    qk.qk_check_device_error()


@pytest.mark.parametrize("kind", ["gauss", "unit", "p3"])
@pytest.mark.parametrize("scene", ["tiny_x", "huge_x", "cancel"])
def test_epilogue_exact_path(qk, orc, kind, scene):
    """Outputs the epilogue's fp32 fast path must hand to its exact fp64 path:
    activations so small that sx 2^e_n could underflow fp32 (every output takes
    the exact path), so large that outputs overflow, and a bias that cancels
    the product of most rows to a small remainder (the fp32 error bound then
    exceeds the distance to the bf16 rounding midpoint).  The result must equal
    the per-group fold route bit for bit either way."""
    M, K, N = 300, 1024, 264
    Wp, s16, o16, allowed = make_weights(orc, kind, N, K, seed=41 + len(kind))
    assert host_plane_count(s16, o16, K) in allowed
    rng = np.random.default_rng(len(scene) * 7 + len(kind))
    xf = rng.standard_normal((M, K)).astype(np.float32)
    b = (rng.standard_normal(N) * 0.1).astype(np.float32)
    if scene == "tiny_x":
        xf *= np.float32(1e-33)
    elif scene == "huge_x":
        xf = np.clip(xf, -1, 1) * np.float32(3.3e38)
    else:
        # rows 0..239 repeat one activation row; the bias is minus that row's
        # output (computed by the oracle without bias), rounded to fp32
        xf[:240] = xf[0]
        y0, _, _, _, _ = orc.w4a8_linear(synthetic.f32_to_bf16_bits(xf[:1]), Wp, s16, o16, None)
        b = -(y0[0].astype(np.uint32) << 16).view(np.float32)
        b = b + (rng.standard_normal(N) * 1e-3 * np.abs(b)).astype(np.float32)
    xb = synthetic.f32_to_bf16_bits(xf)
    _, _, _, y_g, y_f, y_o = run_both_routes(qk, orc, xb, Wp, s16, o16, b, M, K, N)
    assert torch.equal(y_g.view(torch.int16), y_f.view(torch.int16)), (kind, scene)
    if scene == "huge_x":
        assert bool(torch.isinf(y_g.float()).any()), "no output overflowed"
    assert bf16_ulp_distance(t2bits(y_g), y_o).max() <= TOL_ULP
    qk.qk_check_device_error()


def test_epilogue_fast_path_many_outputs(qk, orc):
    """4M outputs of Gaussian weights (two and three digit planes) with a bias:
    about one output in ten thousand lies near enough to a bf16 rounding
    midpoint to take the exact path; every output must equal the fold route's
    bits."""
    M, K, N = 2048, 1024, 2048
    Wp, s16, o16, _ = make_weights(orc, "gauss", N, K, seed=77)
    case = synthetic.LinearCase("fp", M=M, K=K, N=N, bias=True, outlier_frac=0.01, seed=78)
    xb, _, b, _ = case.draw()
    x = to_dev_bf16(xb)
    dw = (to_dev(Wp), dev_fp16(s16), dev_fp16(o16))
    xq, sx, xsum = qk.qk_quantize_activations(x, with_xsum=True)
    y_g = qk.qk_w4a8_gemm(xq, sx, xsum, *dw, to_dev(b), route=GEMM)
    y_f = qk.qk_w4a8_gemm(xq, sx, xsum, *dw, to_dev(b), route=FOLD)
    assert torch.equal(y_g.view(torch.int16), y_f.view(torch.int16))
    qk.qk_check_device_error()


@pytest.mark.parametrize("kind", ["gauss", "unit", "p3", "fold", "negscale"])
def test_prepared_weight(qk, orc, kind):
    """The prepared form (qk_w4a8_prepare once, then the _prepared products)
    gives the same bits as the per-call route for every plane count and the
    fold fallback, on quantized and on bf16 activations, for a small-M (GEMV)
    call too; preparing a second weight into the same (garbage-filled) buffer
    leaves nothing of the first."""
    M, K, N = 300, 1024, 264
    other = "p3" if kind != "p3" else "gauss"
    Wp0, s0, o0, _ = make_weights(orc, other, N, K, seed=91)
    Wp, s16, o16, allowed = make_weights(orc, kind, N, K, seed=90 + len(kind))
    expect = host_plane_count(s16, o16, K)
    dw0 = (to_dev(Wp0), dev_fp16(s0), dev_fp16(o0))
    dw = (to_dev(Wp), dev_fp16(s16), dev_fp16(o16))
    buf = torch.randint(0, 256, (qk.qk_w4a8_prepared_size(N, K),), dtype=torch.uint8,
                        device="cuda")
    qk.qk_w4a8_prepare(*dw0, prepared=buf)
    prepared, planes = qk.qk_w4a8_prepare(*dw, prepared=buf)
    assert planes == (expect if 1 <= expect <= 3 else 255)
    case = synthetic.LinearCase("pr", M=M, K=K, N=N, bias=True, seed=M + N + len(kind))
    xb, _, b, _ = case.draw()
    x = to_dev_bf16(xb)
    bias = to_dev(b)
    y_lin = qk.qk_w4a8_linear(x, *dw, bias)
    y_pre = qk.qk_w4a8_linear_prepared(x, *dw, prepared, bias)
    xq, sx, xsum = qk.qk_quantize_activations(x, with_xsum=True)
    y_gem = qk.qk_w4a8_gemm(xq, sx, xsum, *dw, bias, route=GEMM)
    y_gpr = qk.qk_w4a8_gemm_prepared(xq, sx, xsum, *dw, prepared, bias)
    x8 = x[:8].contiguous()
    y8 = qk.qk_w4a8_linear_prepared(x8, *dw, prepared, bias)
    y8_lin = qk.qk_w4a8_linear(x8, *dw, bias)
    torch.cuda.synchronize()
    for a, c in ((y_pre, y_lin), (y_gpr, y_gem), (y_pre, y_gem), (y8, y8_lin)):
        assert torch.equal(a.view(torch.int16), c.view(torch.int16)), kind
    y_o, _, _, _, _ = orc.w4a8_linear(xb, Wp, s16, o16, b)
    assert bf16_ulp_distance(t2bits(y_pre), y_o).max() <= TOL_ULP
    qk.qk_check_device_error()
