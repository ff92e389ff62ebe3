"""The W8A8 linear with the gated residual epilogue on the GPU against the oracle.

y = bf16(residual + gate * (acc * sx * sw + bias)) evaluated in fp64 and rounded
once; every element within 2 bf16 ulp of the oracle (the tolerance the
epilogue's source page states for its elements), on both W8A8 routes (256 x 256
CTA-pair tiles, and the split-K cluster route for N <= 64), in place and not."""
import numpy as np
import pytest
import torch

from tests.gpu_common import host, qk, t2bits, to_dev, to_dev_bf16  # noqa: F401
from tests.helpers import bf16_ulp_distance, sample_rows
from w4a8_quantized_gemm_token_b200 import synthetic

pytestmark = pytest.mark.gpu

TOL_ULP = 2


def make(qk, orc, case, seed):
    xb, W, b, _ = case.draw()
    Wq_o, sw_o = orc.quant_w8(W)
    Wq, sw = qk.qk_quantize_weights_int8(to_dev(W))
    assert np.array_equal(host(Wq), Wq_o) and np.array_equal(host(sw), sw_o)
    rng = np.random.default_rng(seed)
    gate = (rng.normal(size=case.N) * 0.7).astype(np.float32)
    gate[::7] = 0.0  # some channels closed
    r = synthetic.f32_to_bf16_bits(rng.normal(size=(case.M, case.N)).astype(np.float32) * 2.0)
    return xb, Wq, sw, Wq_o, sw_o, b, gate, r


SHAPES = [(64, 256, 128), (129, 160, 264), (300, 512, 600), (257, 1024, 520),
          # N <= 64: the split-K cluster route
          (300, 992, 40), (1, 5120, 48), (130, 4096, 64)]


@pytest.mark.parametrize("MKN", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("in_place", [False, True], ids=["out", "inplace"])
def test_gated_full_parity(qk, orc, MKN, in_place):
    M, K, N = MKN
    case = synthetic.LinearCase("g", M=M, K=K, N=N, outlier_frac=0.02, bias=(N % 16 == 8),
                                seed=M + 3 * K + N)
    xb, Wq, sw, Wq_o, sw_o, b, gate, r = make(qk, orc, case, seed=M * N)
    x = to_dev_bf16(xb)
    bias = to_dev(b) if b is not None else None
    res = to_dev_bf16(r)
    y = qk.qk_w8a8_linear_gated(x, Wq, sw, bias, to_dev(gate), res, y=res if in_place else None)
    torch.cuda.synchronize()
    out_o, _, _, _ = orc.w8a8_linear_gated(xb, Wq_o, sw_o, b, gate, r)
    d = bf16_ulp_distance(t2bits(y), out_o)
    assert d.max() <= TOL_ULP, f"worst {d.max()} ulp"
    if in_place:
        assert y.data_ptr() == res.data_ptr()
    qk.qk_check_device_error()


def test_gated_closed_gates_return_residual_and_unit_gate_the_linear(qk, orc):
    """gate = 0 returns the residual bit for bit; gate = 1 with a zero residual
    returns exactly what qk_w8a8_linear returns."""
    case = synthetic.LinearCase("gc", M=200, K=768, N=264, seed=31)
    xb, Wq, sw, _, _, b, _, r = make(qk, orc, case, seed=32)
    x, bias = to_dev_bf16(xb), to_dev(b)
    res = to_dev_bf16(r)
    zeros = torch.zeros(case.N, dtype=torch.float32, device="cuda")
    ones = torch.ones(case.N, dtype=torch.float32, device="cuda")
    y0 = qk.qk_w8a8_linear_gated(x, Wq, sw, bias, zeros, res)
    y1 = qk.qk_w8a8_linear_gated(x, Wq, sw, bias, ones, torch.zeros_like(res))
    ylin = qk.qk_w8a8_linear(x, Wq, sw, bias)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), res.view(torch.int16))
    assert torch.equal(y1.view(torch.int16), ylin.view(torch.int16))


def test_gated_dit_attention_projection(qk, orc):
    """The DiT attention projection at full size (4096 x 3072 -> 3072, outlier
    channels, bias) with a gate and a residual: sampled rows against the oracle."""
    case = synthetic.DIT_ATTN
    xb, Wq, sw, Wq_o, sw_o, b, gate, r = make(qk, orc, case, seed=33)
    y = qk.qk_w8a8_linear_gated(to_dev_bf16(xb), Wq, sw, to_dev(b), to_dev(gate), to_dev_bf16(r))
    torch.cuda.synchronize()
    rows = sample_rows(case.M, extra=6, seed=7)
    xq_o, sx_o = orc.quant_act(xb[rows])
    acc_o = orc.w8a8_acc(xq_o, Wq_o)
    out_o = orc.w8a8_gated(acc_o, sx_o, sw_o, b, gate, r[rows])
    d = bf16_ulp_distance(t2bits(y[torch.from_numpy(rows).cuda()]), out_o)
    print(f"gated attn: rows={len(rows)} worst={d.max()} ulp")
    assert d.max() <= TOL_ULP
    qk.qk_check_device_error()


def test_gated_rejects_missing_operands(qk):
    x = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros(16, 64, dtype=torch.int8, device="cuda")
    sw = torch.ones(16, dtype=torch.float32, device="cuda")
    res = torch.zeros(8, 16, dtype=torch.bfloat16, device="cuda")
    lib = qk.lib
    st = lib.qk_w8a8_linear_gated(x.data_ptr(), 8, 64, Wq.data_ptr(), sw.data_ptr(), None, None,
                                  res.data_ptr(), 16, res.data_ptr(), None, 0, None)
    assert st == 1  # QK_ERR_INVALID_ARG: no gate
