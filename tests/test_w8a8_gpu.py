"""The W8A8 linear on the GPU against the oracle.

int32 accumulators bit-exact (through the accumulator hook, same mainloop);
bf16 outputs within 2 bf16 ulp of the oracle's fp64 dequant rounded to bf16.
Small shapes compare every output; the DiT configs compare sampled rows that
cover tile edges and the ragged tail, computed one by one by the oracle."""
import numpy as np
import pytest
import torch

from tests.gpu_common import host, qk, t2bits, to_dev, to_dev_bf16  # noqa: F401
from tests.helpers import bf16_ulp_distance, sample_rows
from w4a8_quantized_gemm_token_b200 import synthetic

pytestmark = pytest.mark.gpu

TOL_ULP = 2

SHAPES = [  # (M, K, N): tiles of 128 x 256 with K blocks of 128
    # the one-kernel form (qk_w8a8_linear_fused: the GEMM's epilogue warps
    # quantize x): 8192 x 256 x 72 has 64 row blocks behind one column of
    # tiles; 600 x 8192 has rows longer than 4096 elements (two passes per row)
    (8192, 256, 72),
    (600, 8192, 264),
    (2, 4096, 4096),
    (64, 256, 128),
    (1, 32, 8),
    (3, 96, 24),
    (129, 160, 264),
    (300, 512, 600),
    (257, 1024, 520),
    (128, 128, 256),
    (513, 384, 776),
    # N <= 64: the split-K cluster route (K ranges over 1, 2, 4 or 8 CTAs,
    # ragged M, N and K blocks)
    (300, 992, 40),
    (1, 5120, 48),
    (130, 4096, 64),
    (129, 384, 16),
]


def prepare(qk, orc, case):
    xb, W, b, _ = case.draw()
    Wq_o, sw_o = orc.quant_w8(W)
    Wq, sw = qk.qk_quantize_weights_int8(to_dev(W))
    assert np.array_equal(host(Wq), Wq_o) and np.array_equal(host(sw), sw_o)
    return xb, Wq, sw, Wq_o, sw_o, b


@pytest.mark.parametrize("MKN", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("with_bias", [True, False])
def test_w8a8_small_full_parity(qk, orc, MKN, with_bias):
    M, K, N = MKN
    case = synthetic.LinearCase("s", M=M, K=K, N=N, outlier_frac=0.02, bias=with_bias, seed=M + K + N)
    xb, Wq, sw, Wq_o, sw_o, b = prepare(qk, orc, case)
    x = to_dev_bf16(xb)
    bias = to_dev(b) if with_bias else None
    y = qk.qk_w8a8_linear(x, Wq, sw, bias)
    ws = torch.empty(qk.qk_w8a8_workspace_size(M, K), dtype=torch.uint8, device="cuda")
    yf = qk.qk_w8a8_linear(x, Wq, sw, bias, workspace=ws, fused=True)
    xq, sx, _ = qk.qk_quantize_activations(x)
    acc = qk.qk_debug_w8a8_acc(xq, Wq)
    torch.cuda.synchronize()
    y_o, xq_o, sx_o, acc_o = orc.w8a8_linear(xb, Wq_o, sw_o, b)
    assert np.array_equal(host(xq), xq_o) and np.array_equal(host(sx), sx_o)
    assert np.array_equal(host(acc).astype(np.int64), acc_o)
    d = bf16_ulp_distance(t2bits(y), y_o)
    assert d.max() <= TOL_ULP, f"worst {d.max()} ulp"
    # the one-kernel form: the same bits, and the same codes and scales left
    # in the workspace
    assert torch.equal(yf.view(torch.int16), y.view(torch.int16))
    off = (M * K + 255) // 256 * 256
    assert np.array_equal(host(ws[: M * K].view(torch.int8).view(M, K)), xq_o)
    assert np.array_equal(host(ws[off: off + 4 * M].view(torch.float32)), sx_o)
    qk.qk_check_device_error()


@pytest.mark.parametrize("case", [synthetic.TINY, synthetic.DIT_ATTN, *synthetic.SWEEP,
                                  synthetic.DIT_MLP, synthetic.QUICKSTART[0]],
                         ids=lambda c: c.name)
def test_w8a8_configs(qk, orc, case):
    """Every DiT config at full size: all codes bit-exact, accumulators and
    outputs of sampled rows against the oracle."""
    xb, Wq, sw, Wq_o, sw_o, b = prepare(qk, orc, case)
    x = to_dev_bf16(xb)
    bias = to_dev(b) if b is not None else None
    ws = torch.empty(qk.qk_w8a8_workspace_size(case.M, case.K), dtype=torch.uint8, device="cuda")
    y = qk.qk_w8a8_linear(x, Wq, sw, bias, workspace=ws)
    yf = qk.qk_w8a8_linear(x, Wq, sw, bias, workspace=ws, fused=True)  # one-kernel form
    xq, sx, _ = qk.qk_quantize_activations(x)
    acc = qk.qk_debug_w8a8_acc(xq, Wq)
    torch.cuda.synchronize()
    assert torch.equal(yf.view(torch.int16), y.view(torch.int16))
    rows = np.arange(case.M) if case.M <= 256 else sample_rows(case.M, extra=6, seed=case.M)
    xq_all, sx_all = orc.quant_act(xb)
    assert np.array_equal(host(xq), xq_all) and np.array_equal(host(sx), sx_all)
    acc_o = orc.w8a8_acc(xq_all[rows], Wq_o)
    rows_t = torch.from_numpy(rows).cuda()
    assert np.array_equal(host(acc[rows_t]).astype(np.int64), acc_o)
    y_o = orc.w8a8_dequant(acc_o, sx_all[rows], sw_o, b)
    d = bf16_ulp_distance(t2bits(y[rows_t]), y_o)
    hist = np.bincount(d.ravel(), minlength=3)
    print(f"{case.name}: rows={len(rows)} worst={d.max()} ulp histogram={hist.tolist()}")
    assert d.max() <= TOL_ULP
    qk.qk_check_device_error()


def test_w8a8_deterministic_and_api_variants(qk, orc):
    case = synthetic.LinearCase("d", M=777, K=1024, N=1032, outlier_frac=0.01, seed=5)
    xb, Wq, sw, _, _, b = prepare(qk, orc, case)
    x = to_dev_bf16(xb)
    bias = to_dev(b)
    y1 = qk.qk_w8a8_linear(x, Wq, sw, bias)                       # library-owned workspace
    ws = torch.empty(qk.qk_w8a8_workspace_size(777, 1024), dtype=torch.uint8, device="cuda")
    y2 = qk.qk_w8a8_linear(x, Wq, sw, bias, workspace=ws)
    xq, sx, _ = qk.qk_quantize_activations(x)
    y3 = qk.qk_w8a8_gemm(xq, sx, Wq, sw, bias)                    # split API
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())  # the same workspace: not concurrently
    with torch.cuda.stream(s):
        y4 = qk.qk_w8a8_linear(x, Wq, sw, bias, workspace=ws)     # another stream
    s.synchronize()
    torch.cuda.synchronize()
    for y in (y2, y3, y4):
        assert torch.equal(y1.view(torch.int16), y.view(torch.int16))
    # the one-kernel route leaves the activation codes and scales in the workspace
    wq = ws[: 777 * 1024].view(torch.int8).view(777, 1024)
    off = (777 * 1024 + 255) // 256 * 256
    wsx = ws[off: off + 777 * 4].view(torch.float32)
    assert torch.equal(wq, xq) and torch.equal(wsx.view(torch.int32), sx.view(torch.int32))


@pytest.mark.parametrize("MKN", [(200, 256, 264), (200, 1024, 40)], ids=["tiles", "splitk"])
def test_w8a8_guard_bands(qk, orc, MKN):
    """Outputs land only inside y: a sentinel halo around it stays untouched."""
    M, K, N = MKN
    case = synthetic.LinearCase("g", M=M, K=K, N=N, seed=9)
    xb, Wq, sw, _, _, b = prepare(qk, orc, case)
    pad = 4096
    flat = torch.full((M * N + 2 * pad,), 0x7FBF, dtype=torch.int16, device="cuda")
    y = flat[pad: pad + M * N].view(M, N).view(torch.bfloat16)
    qk.qk_w8a8_linear(to_dev_bf16(xb), Wq, sw, to_dev(b), y=y)
    torch.cuda.synchronize()
    assert bool((flat[:pad] == 0x7FBF).all()) and bool((flat[-pad:] == 0x7FBF).all())
    assert not bool((flat[pad: pad + M * N] == 0x7FBF).any())


def test_w8a8_fused_workspace_reuse_and_garbage(qk, orc):
    """The one-kernel W8A8 linear keeps a readiness word per row in the
    workspace, set to each launch's own value: a workspace full of garbage, or
    left by a call of another shape, gives the same bits as the two-kernel
    linear."""
    cases = [synthetic.LinearCase("wa", M=700, K=1024, N=520, seed=41),
             synthetic.LinearCase("wb", M=1300, K=512, N=264, seed=42)]
    prepared = [prepare(qk, orc, c) for c in cases]
    need = max(qk.qk_w8a8_workspace_size(c.M, c.K) for c in cases)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    fresh = [qk.qk_w8a8_linear(to_dev_bf16(p[0]), p[1], p[2], to_dev(p[5])) for p in prepared]
    for rep in range(2):
        for p, want in zip(prepared, fresh):
            y = qk.qk_w8a8_linear(to_dev_bf16(p[0]), p[1], p[2], to_dev(p[5]), workspace=ws,
                                  fused=True)
            torch.cuda.synchronize()
            assert torch.equal(y.view(torch.int16), want.view(torch.int16))
    y_o, _, _, _ = orc.w8a8_linear(prepared[0][0], prepared[0][3], prepared[0][4], prepared[0][5])
    assert bf16_ulp_distance(t2bits(fresh[0]), y_o).max() <= TOL_ULP
    qk.qk_check_device_error()


def test_w8a8_zero_rows_and_integer_closed_form(qk, orc):
    """Integer inputs with row absmax 127 reproduce the exact integer GEMM; a
    zero row outputs bf16(bias)."""
    rng = np.random.default_rng(3)
    M, K, N = 130, 256, 136
    x = rng.integers(-127, 128, size=(M, K)).astype(np.float32)
    x[:, 5] = 127
    x[7] = 0.0
    W = rng.integers(-127, 128, size=(N, K)).astype(np.float32)
    W[:, 9] = -127
    b = rng.integers(-500, 500, size=N).astype(np.float32)
    from tests.test_oracle_pins import bf16_bits

    xb = bf16_bits(x)
    Wq, sw = qk.qk_quantize_weights_int8(to_dev(W))
    y = qk.qk_w8a8_linear(to_dev_bf16(xb), Wq, sw, to_dev(b))
    exact = (x.astype(np.int64) @ W.astype(np.int64).T + b.astype(np.int64)).astype(np.float32)
    want = torch.from_numpy(exact).to(torch.bfloat16)
    assert torch.equal(y.cpu().view(torch.int16), want.view(torch.int16))


@pytest.mark.parametrize("MKN", [(130, 65536, 264), (8, 65536, 16)], ids=["tiles", "splitk"])
def test_w8a8_max_k_saturated_codes(qk, orc, MKN):
    """K = 65536, the contract's maximum, with every code at +-127 (x rows and W
    rows of +-1): the int32 accumulators reach +-127^2 * 65536 = 1 057 030 144,
    just below 2^31, exactly, and the outputs match the oracle."""
    M, K, N = MKN
    xs = np.where(np.arange(M)[:, None] % 2 == 0, 1.0, -1.0) * np.ones((M, K))
    ws = np.where(np.arange(N)[:, None] % 3 == 0, -1.0, 1.0) * np.ones((N, K))
    xb = synthetic.f32_to_bf16_bits(xs.astype(np.float32))
    W = ws.astype(np.float32)
    Wq_o, sw_o = orc.quant_w8(W)
    Wq, sw = qk.qk_quantize_weights_int8(to_dev(W))
    assert np.array_equal(host(Wq), Wq_o)
    x = to_dev_bf16(xb)
    y = qk.qk_w8a8_linear(x, Wq, sw)
    xq, sx, _ = qk.qk_quantize_activations(x)
    acc = qk.qk_debug_w8a8_acc(xq, Wq)
    torch.cuda.synchronize()
    want = (np.sign(xs[:, :1]) * np.sign(ws[:, 0])[None, :]) * 127 * 127 * K
    assert np.array_equal(host(acc).astype(np.int64), want.astype(np.int64))
    xq_o, sx_o = orc.quant_act(xb)
    y_o = orc.w8a8_dequant(orc.w8a8_acc(xq_o, Wq_o), sx_o, sw_o, None)
    assert bf16_ulp_distance(t2bits(y), y_o).max() <= TOL_ULP
    qk.qk_check_device_error()
