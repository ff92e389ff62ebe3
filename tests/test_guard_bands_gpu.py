"""Guard bands for every output writer: each output tensor sits inside a larger
buffer whose halo before and after it holds a sentinel bf16 pattern (a NaN,
which no finite output takes).  After the call the halo must be untouched and
no sentinel may remain inside the output.  This stands in for a memory
checker: the stores most likely to stray are those of ragged last CTAs, of the
TMA stores that clip the M and N edges, and of the rows finalized after the
cross-CTA reductions in distributed shared memory."""
import numpy as np
import pytest
import torch

from tests.gpu_common import host, qk, to_dev, to_dev_bf16  # noqa: F401
from w4a8_quantized_gemm_token_b200 import synthetic

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FBF   # a bf16 NaN
PAD = 4096          # elements of halo on each side


def haloed(shape):
    """(flat int16 buffer, bf16 view of `shape` in its middle)."""
    n = int(np.prod(shape))
    flat = torch.full((n + 2 * PAD,), SENTINEL, dtype=torch.int16, device="cuda")
    return flat, flat[PAD: PAD + n].view(*shape).view(torch.bfloat16)


def assert_halo_intact(flat):
    torch.cuda.synchronize()
    assert bool((flat[:PAD] == SENTINEL).all()), "a store landed before the output"
    assert bool((flat[-PAD:] == SENTINEL).all()), "a store landed after the output"
    assert not bool((flat[PAD:-PAD] == SENTINEL).any()), "an output element was not written"


def w4_weights(qk, K, N, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    return qk.qk_quantize_weights_int4(to_dev(W))


def x_dev(M, K, seed):
    case = synthetic.LinearCase("gb", M=M, K=K, N=8, bias=False, seed=seed)
    xb, _, _, _ = case.draw()
    return to_dev_bf16(xb)


# Every GEMV tiling the host picks: one-token dp4a kernel (1 to 4 chunks per
# lane, ragged last CTA), clusters of 1, 2 and 4 CTAs, 32-row CTAs with a ragged
# last CTA, a partial last group range, in-kernel and separate quantization.
GEMV_SHAPES = [(1, 64, 8), (1, 1024, 264), (1, 3072, 136), (1, 2048, 40), (3, 192, 40),
               (11, 1024, 264), (16, 3072, 128), (5, 640, 2056), (9, 1024, 2376),
               (12, 2112, 136), (8, 4096, 4096), (16, 4096, 4096)]


@pytest.mark.parametrize("MKN", GEMV_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_gemv_guard_bands(qk, MKN):
    M, K, N = MKN
    Wp, s, o = w4_weights(qk, K, N, seed=K + N)
    bias = to_dev(np.linspace(-1, 1, N).astype(np.float32))
    x = x_dev(M, K, seed=M + K)
    flat, y = haloed((M, N))
    qk.qk_w4a8_linear(x, Wp, s, o, bias, y=y)              # the public call (its own plan)
    assert_halo_intact(flat)
    xq, sx, xsum = qk.qk_quantize_activations(x, with_xsum=True)
    flat2, y2 = haloed((M, N))
    qk.qk_w4a8_gemm(xq, sx, xsum, Wp, s, o, bias, y=y2, route=2)   # GEMV on xq
    assert_halo_intact(flat2)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    qk.qk_check_device_error()


@pytest.mark.parametrize("MKN", [(17, 64, 8), (17, 192, 72), (129, 192, 72), (300, 1024, 264),
                                 (257, 320, 64), (16, 256, 136)],
                         ids=lambda s: "x".join(map(str, s)))
def test_w4a8_gemm_guard_bands(qk, MKN):
    M, K, N = MKN
    Wp, s, o = w4_weights(qk, K, N, seed=K * 3 + N)
    bias = to_dev(np.linspace(-2, 2, N).astype(np.float32))
    x = x_dev(M, K, seed=M * 5 + K)
    xq, sx, xsum = qk.qk_quantize_activations(x, with_xsum=True)
    flat, y = haloed((M, N))
    qk.qk_w4a8_gemm(xq, sx, xsum, Wp, s, o, bias, y=y, route=1)
    assert_halo_intact(flat)
    if M > 16:
        flat2, y2 = haloed((M, N))
        qk.qk_w4a8_linear(x, Wp, s, o, bias, y=y2)
        assert_halo_intact(flat2)
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    qk.qk_check_device_error()


@pytest.mark.parametrize("MKN", [(200, 256, 264), (77, 1024, 40), (1, 512, 8)],
                         ids=["tiles", "splitk", "one_row"])
def test_w8a8_gated_guard_bands(qk, MKN):
    M, K, N = MKN
    rng = np.random.default_rng(M + K + N)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Wq, sw = qk.qk_quantize_weights_int8(to_dev(W))
    bias = to_dev((rng.standard_normal(N) * 0.1).astype(np.float32))
    gate = to_dev((rng.standard_normal(N) * 0.5).astype(np.float32))
    res = to_dev_bf16(synthetic.f32_to_bf16_bits(rng.standard_normal((M, N)).astype(np.float32)))
    x = x_dev(M, K, seed=M * 7 + K)
    flat, y = haloed((M, N))
    qk.qk_w8a8_linear_gated(x, Wq, sw, bias, gate, res, y=y)
    assert_halo_intact(flat)
    qk.qk_check_device_error()


@pytest.mark.parametrize("BHL", [(1, 3, 1000), (2, 1, 200), (1, 1, 8)],
                         ids=lambda s: "x".join(map(str, s)))
def test_sage_attention_guard_bands(qk, BHL):
    B, H, L = BHL
    rng = np.random.default_rng(B * 100 + H * 10 + L)

    def t():
        return to_dev_bf16(synthetic.f32_to_bf16_bits(
            rng.standard_normal((B, H, L, 128)).astype(np.float32)))

    q, k, v = t(), t(), t()
    flat, out = haloed((B, H, L, 128))
    qk.qk_sage_attention(q, k, v, scale=128 ** -0.5, out=out)
    assert_halo_intact(flat)
    qk.qk_check_device_error()
