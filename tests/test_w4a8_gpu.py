"""The W4A8 linear on the GPU against the oracle.

Per-group int32 accumulators bit-exact on both routes (weight-streaming GEMV for
M <= 16, tcgen05 GEMM otherwise); bf16 outputs within 2 bf16 ulp of the
oracle's fp64 fold rounded to bf16; the two routes agree where both apply."""
import numpy as np
import pytest
import torch

from tests.gpu_common import host, qk, t2bits, to_dev, to_dev_bf16  # noqa: F401
from tests.helpers import bf16_ulp_distance, sample_rows
from w4a8_quantized_gemm_token_b200 import synthetic

pytestmark = pytest.mark.gpu

TOL_ULP = 2
GEMV, GEMM = 2, 1


def prepare(qk, orc, case):
    xb, W, b, _ = case.draw()
    Wp_o, s_o, o_o = orc.quant_w4(W)
    Wp, s, o = qk.qk_quantize_weights_int4(to_dev(W))
    assert np.array_equal(host(Wp), Wp_o)
    assert np.array_equal(t2bits(s), s_o) and np.array_equal(t2bits(o), o_o)
    return xb, (Wp, s, o), (Wp_o, s_o, o_o), b


# 9 x 1024 x 2376: 32-row CTAs with a ragged last CTA.  qk_w4a8_linear
# quantizes x inside the GEMV for up to 8 tokens when one CTA's K slice of x
# fits its registers; 9 tokens and more, 16 x 3072 x 128 and 12 x 2112 x 136
# take the quantization kernel + GEMV (2112 = 33 groups: a partial last group
# range).
GEMV_SHAPES = [(1, 64, 8), (1, 4096, 4096), (8, 4096, 4096), (16, 4096, 4096), (3, 192, 40),
               (11, 1024, 264), (16, 3072, 128), (5, 640, 2056), (9, 1024, 2376),
               (12, 2112, 136),
               # one token, K a multiple of 1024: the dp4a kernel (1 to 4 chunks per
               # lane, ragged last CTA)
               (1, 1024, 264), (1, 3072, 136), (1, 2048, 40)]


@pytest.mark.parametrize("MKN", GEMV_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_gemv_group_acc_and_output(qk, orc, MKN):
    M, K, N = MKN
    case = synthetic.LinearCase("v", M=M, K=K, N=N, bias=(N % 16 == 8), seed=M * 31 + K + N)
    xb, dev_w, ora_w, b = prepare(qk, orc, case)
    x = to_dev_bf16(xb)
    xq, sx, xsum = qk.qk_quantize_activations(x, with_xsum=True)
    acc = qk.qk_debug_w4a8_group_acc(xq, dev_w[0], 0, M, GEMV)
    bias = to_dev(b) if b is not None else None
    y = qk.qk_w4a8_linear(x, *dev_w, bias)
    y2 = qk.qk_w4a8_gemm(xq, sx, xsum, *dev_w, bias, route=GEMV)
    torch.cuda.synchronize()
    y_o, xq_o, sx_o, xsum_o, acc_o = orc.w4a8_linear(xb, *ora_w, b)
    assert np.array_equal(host(xq), xq_o) and np.array_equal(host(xsum), xsum_o)
    assert np.array_equal(host(acc).astype(np.int64), acc_o)
    d = bf16_ulp_distance(t2bits(y), y_o)
    assert d.max() <= TOL_ULP, f"worst {d.max()} ulp"
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    qk.qk_check_device_error()


@pytest.mark.parametrize("K", [1024, 4096])
def test_one_token_quantization_ties(qk, orc, K):
    """The one-token GEMV quantizes bf16 x itself.  A row whose absmax is 127
    has the multiplier 1, so values k + 1/2 sit exactly on rounding ties: its
    output must equal, bit for bit, the product on the codes of the stand-alone
    quantization kernel (which match the oracle), and the oracle within 2 ulp."""
    N = 264
    case = synthetic.LinearCase("ties", M=1, K=K, N=N, bias=True, seed=K + 5)
    _, dev_w, ora_w, b = prepare(qk, orc, case)
    rng = np.random.default_rng(K)
    halves = np.arange(127, dtype=np.float32) + np.float32(0.5)            # 0.5 .. 126.5
    vals = np.concatenate([halves, -halves, np.arange(-127, 128, dtype=np.float32)])
    row = rng.choice(vals, size=K).astype(np.float32)
    row[rng.integers(0, K)] = 127.0
    xb = synthetic.f32_to_bf16_bits(row[None, :])
    assert np.array_equal((xb.astype(np.uint32) << 16).view(np.float32), row[None, :])  # exact in bf16
    x = to_dev_bf16(xb)
    xq, sx, xsum = qk.qk_quantize_activations(x, with_xsum=True)
    bias = to_dev(b)
    y = qk.qk_w4a8_linear(x, *dev_w, bias)
    y2 = qk.qk_w4a8_gemm(xq, sx, xsum, *dev_w, bias, route=GEMV)
    torch.cuda.synchronize()
    y_o, xq_o, sx_o, _, _ = orc.w4a8_linear(xb, *ora_w, b)
    assert float(sx_o[0]) == 1.0
    assert np.array_equal(host(xq), xq_o)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    assert bf16_ulp_distance(t2bits(y), y_o).max() <= TOL_ULP
    qk.qk_check_device_error()


@pytest.mark.parametrize("case", synthetic.W4A8[:3], ids=lambda c: c.name)
def test_w4a8_gemv_configs(qk, orc, case):
    xb, dev_w, ora_w, b = prepare(qk, orc, case)
    y = qk.qk_w4a8_linear(to_dev_bf16(xb), *dev_w)
    torch.cuda.synchronize()
    y_o, _, _, _, _ = orc.w4a8_linear(xb, *ora_w, None)
    d = bf16_ulp_distance(t2bits(y), y_o)
    print(f"{case.name}: worst={d.max()} ulp histogram={np.bincount(d.ravel(), minlength=3).tolist()}")
    assert d.max() <= TOL_ULP


def test_gemv_deterministic(qk, orc):
    case = synthetic.LinearCase("det", M=16, K=4096, N=4096, bias=False, seed=77)
    xb, dev_w, _, _ = prepare(qk, orc, case)
    x = to_dev_bf16(xb)
    ys = [qk.qk_w4a8_linear(x, *dev_w) for _ in range(3)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(ys[0].view(torch.int16), y.view(torch.int16))


GEMM_SHAPES = [(17, 64, 8), (129, 192, 72), (300, 1024, 264), (64, 4096, 136), (257, 320, 64),
               (16, 256, 128),
               # K = 65536, the contract's maximum: 1024 groups folded per output
               (40, 65536, 72)]


@pytest.mark.parametrize("MKN", GEMM_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_gemm_group_acc_and_output(qk, orc, MKN):
    M, K, N = MKN
    case = synthetic.LinearCase("m", M=M, K=K, N=N, bias=(N % 16 == 8), seed=M * 17 + K + N)
    xb, dev_w, ora_w, b = prepare(qk, orc, case)
    x = to_dev_bf16(xb)
    xq, sx, xsum = qk.qk_quantize_activations(x, with_xsum=True)
    acc = qk.qk_debug_w4a8_group_acc(xq, dev_w[0], 0, M, GEMM)
    bias = to_dev(b) if b is not None else None
    y = qk.qk_w4a8_gemm(xq, sx, xsum, *dev_w, bias, route=GEMM)
    torch.cuda.synchronize()
    y_o, xq_o, sx_o, xsum_o, acc_o = orc.w4a8_linear(xb, *ora_w, b)
    assert np.array_equal(host(acc).astype(np.int64), acc_o)
    d = bf16_ulp_distance(t2bits(y), y_o)
    assert d.max() <= TOL_ULP, f"worst {d.max()} ulp"
    if M > 16:  # the public call takes the GEMM route
        y2 = qk.qk_w4a8_linear(x, *dev_w, bias)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    qk.qk_check_device_error()


@pytest.mark.parametrize("case, blocks", [
    (synthetic.W4A8[3], [(0, 4), (126, 130), (2047, 2051), (4092, 4096)]),
    # the README's quick-start matmul: ragged M (14040 = 109 tiles of 128 + 88)
    (synthetic.QUICKSTART[1], [(0, 4), (126, 130), (7040, 7044), (13950, 13954), (14036, 14040)]),
], ids=lambda v: v.name if hasattr(v, "name") else "")
def test_w4a8_gemm_config(qk, orc, case, blocks):
    """A large-M W4A8 workload: every code bit-exact, per-group sums and
    outputs of sampled row blocks (first, last, tile edges) against the oracle."""
    xb, dev_w, ora_w, _ = prepare(qk, orc, case)
    x = to_dev_bf16(xb)
    y = qk.qk_w4a8_linear(x, *dev_w)
    xq, sx, xsum = qk.qk_quantize_activations(x, with_xsum=True)
    torch.cuda.synchronize()
    xq_o, sx_o = orc.quant_act(xb)
    assert np.array_equal(host(xq), xq_o) and np.array_equal(host(sx), sx_o)
    worst = 0
    for m0, m1 in blocks:
        acc = qk.qk_debug_w4a8_group_acc(xq, dev_w[0], m0, m1, GEMM)
        torch.cuda.synchronize()
        acc_o = orc.w4a8_group_acc(xq_o[m0:m1], ora_w[0])
        assert np.array_equal(host(acc).astype(np.int64), acc_o)
        y_o = orc.w4a8_dequant(acc_o, orc.group_sums(xq_o[m0:m1]), sx_o[m0:m1], ora_w[1], ora_w[2])
        d = bf16_ulp_distance(t2bits(y[m0:m1]), y_o)
        worst = max(worst, int(d.max()))
    print(f"{case.name}: sampled worst={worst} ulp")
    assert worst <= TOL_ULP


def test_routes_agree_at_m16(qk, orc):
    """At M = 16 both routes apply: identical per-group integers, outputs equal
    up to the fp64 summation order (at most 1 ulp)."""
    case = synthetic.LinearCase("r", M=16, K=4096, N=1024, bias=True, seed=3)
    xb, dev_w, _, b = prepare(qk, orc, case)
    xq, sx, xsum = qk.qk_quantize_activations(to_dev_bf16(xb), with_xsum=True)
    a_v = qk.qk_debug_w4a8_group_acc(xq, dev_w[0], 0, 16, GEMV)
    a_m = qk.qk_debug_w4a8_group_acc(xq, dev_w[0], 0, 16, GEMM)
    y_v = qk.qk_w4a8_gemm(xq, sx, xsum, *dev_w, to_dev(b), route=GEMV)
    y_m = qk.qk_w4a8_gemm(xq, sx, xsum, *dev_w, to_dev(b), route=GEMM)
    torch.cuda.synchronize()
    assert torch.equal(a_v, a_m)
    assert bf16_ulp_distance(t2bits(y_v), t2bits(y_m)).max() <= 1


def test_large_k_small_m_routes_to_gemm(qk, orc):
    """M <= 16 with a K whose GEMV tiling does not fit the registers: the
    explicit GEMV route is refused, the automatic route takes the GEMM."""
    # K = 32768: every tiling leaves a warp more than 16 groups of its rows
    case = synthetic.LinearCase("lk", M=4, K=32768, N=64, bias=True, seed=8)
    xb, dev_w, ora_w, b = prepare(qk, orc, case)
    x = to_dev_bf16(xb)
    xq, sx, xsum = qk.qk_quantize_activations(x, with_xsum=True)
    with pytest.raises(qk.QKError) as e:
        qk.qk_w4a8_gemm(xq, sx, xsum, *dev_w, to_dev(b), route=GEMV)
    assert e.value.status == 2
    y = qk.qk_w4a8_linear(x, *dev_w, to_dev(b))
    torch.cuda.synchronize()
    y_o, _, _, _, _ = orc.w4a8_linear(xb, *ora_w, b)
    assert bf16_ulp_distance(t2bits(y), y_o).max() <= TOL_ULP
