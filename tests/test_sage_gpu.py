"""INT8 attention (the sage_attention bullet of the qlip-mlx README) on the GPU
against the oracle.

The kernel evaluates scores and the softmax in fp32 and feeds P V with the
weights rounded to bf16 (normalised by the sum of the rounded weights), then
rounds the output to bf16.  Each weight then carries a relative error of at
most 2^-9 (bf16) plus ~2^-21 (fp32 score arithmetic, the 2^x approximation),
so the weighted mean moves by at most ~2^-8 max_j |v_j|, and the two bf16
roundings (the kernel's and the oracle's) add 2^-8 |o|.  The test bound per
element is |o_gpu - o_exact| <= 2^-8 (max_j |v_j| + |o_exact|) + 2^-20, with
o_exact the oracle's fp64 output (before its rounding)."""
import numpy as np
import pytest
import torch

from tests.gpu_common import qk, t2bits  # noqa: F401
from w4a8_quantized_gemm_token_b200 import synthetic

pytestmark = pytest.mark.gpu


def bf16_val(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def draw(B, H, L, seed, q_scale=1.0):
    rng = np.random.default_rng(seed)
    q = synthetic.f32_to_bf16_bits((rng.standard_normal((B, H, L, 128)) * q_scale).astype(np.float32))
    k = synthetic.f32_to_bf16_bits(rng.standard_normal((B, H, L, 128)).astype(np.float32))
    v = synthetic.f32_to_bf16_bits(rng.standard_normal((B, H, L, 128)).astype(np.float32))
    return q, k, v


def to_dev(bits):
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def check(out_bits, o64, v_bits):
    got = bf16_val(out_bits).astype(np.float64)
    vmax = np.abs(bf16_val(v_bits)).max(axis=-2, keepdims=True).astype(np.float64)  # per head
    bound = 2.0 ** -8 * (vmax + np.abs(o64)) + 2.0 ** -20
    err = np.abs(got - o64)
    worst = (err / bound).max()
    assert np.isfinite(got).all()
    assert worst <= 1.0, f"worst error / bound = {worst:.3f}"
    return float(err.max()), float(worst)


SHAPES = [(1, 1, 128), (1, 2, 256), (2, 1, 200), (1, 1, 8), (1, 3, 1000), (1, 1, 1024)]


@pytest.mark.parametrize("BHL", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_sage_attention_parity(qk, orc, BHL):
    B, H, L = BHL
    q, k, v = draw(B, H, L, seed=B * 1000 + H * 100 + L, q_scale=2.0)
    out = qk.qk_sage_attention(to_dev(q), to_dev(k), to_dev(v), scale=128 ** -0.5)
    torch.cuda.synchronize()
    qk.qk_check_device_error()
    ref, o64 = orc.sage_attention(q, k, v, 128 ** -0.5, with_f64=True)
    err, worst = check(t2bits(out), o64, v)
    exact = np.mean(t2bits(out) == ref)
    print(f"sage {BHL}: max |err| {err:.2e}, worst/bound {worst:.3f}, bf16-equal {exact:.3f}")


def test_sage_attention_scale_and_peaked_rows(qk, orc):
    """A large scale (peaked softmax, one key dominating many rows) and scale 0
    (uniform weights: the mean of v)."""
    B, H, L = 1, 2, 384
    q, k, v = draw(B, H, L, seed=7, q_scale=4.0)
    for scale in (1.0, 0.0):
        out = qk.qk_sage_attention(to_dev(q), to_dev(k), to_dev(v), scale=scale)
        torch.cuda.synchronize()
        _, o64 = orc.sage_attention(q, k, v, scale, with_f64=True)
        check(t2bits(out), o64, v)


def test_sage_attention_deterministic_and_workspace(qk):
    B, H, L = 1, 2, 512
    q, k, v = (to_dev(t) for t in draw(B, H, L, seed=9))
    o1 = qk.qk_sage_attention(q, k, v)
    ws = torch.empty(qk.qk_sage_attention_workspace_size(B, H, L), dtype=torch.uint8, device="cuda")
    o2 = qk.qk_sage_attention(q, k, v, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


def test_sage_attention_quickstart_heads_sampled(qk, orc):
    """The README's quick-start attention shape (40 heads x 14040 tokens, head
    dim 128): sampled query rows of a few heads against the oracle (every key)."""
    B, H, L = 1, 40, 14040
    q, k, v = draw(B, H, L, seed=11)
    out = qk.qk_sage_attention(to_dev(q), to_dev(k), to_dev(v), scale=128 ** -0.5)
    torch.cuda.synchronize()
    qk.qk_check_device_error()
    ob = t2bits(out)
    rows = np.array([0, 1, 127, 128, 7000, 13951, 13952, 14039])
    for h in (0, 17, 39):
        _, o64 = orc.sage_attention_rows(q[0, h], k[0, h], v[0, h], 128 ** -0.5, rows)
        check(ob[0, h][rows], o64, v[0, h][None])


def test_sage_attention_rejects_bad_shapes(qk):
    x = torch.zeros(1, 1, 12, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(qk.QKError):
        qk.qk_sage_attention(x, x, x)  # L % 8 != 0
    y = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(qk.QKError):
        qk.qk_sage_attention(y, y, y)  # head dim 64
    z = torch.zeros(1, 1, 16, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(qk.QKError):
        qk.qk_sage_attention(z, z, z, scale=-1.0)  # negative scale
