"""Quantization kernels on the GPU against the oracle: codes, scales and group
sums bit-exact (activations per token, W8 per channel, W4 affine group 64)."""
import json
import os

import numpy as np
import pytest
import torch

from tests.gpu_common import host, qk, t2bits, to_dev, to_dev_bf16  # noqa: F401
from w4a8_quantized_gemm_token_b200 import synthetic

pytestmark = pytest.mark.gpu

MS = [1, 2, 3, 15, 16, 17, 63, 64, 65, 129]
# one warp per row (K <= 2048), then 2, 4 or 8 warps per row with 5..8 chunks
# per thread (2112 .. 16384, including K % 64 != 0 without group sums), then
# the two-pass kernel (20480)
KS = [32, 64, 96, 160, 2048, 2112, 3072, 3104, 3584, 4096, 5120, 6144, 7168, 8192, 10240,
      12288, 16384, 20480]


@pytest.mark.parametrize("K", KS)
def test_act_quant_bit_exact(qk, orc, K):
    for M in MS:
        case = synthetic.LinearCase("q", M=M, K=K, N=8, outlier_frac=0.01, seed=M * 7 + K)
        xb, _, _, _ = case.draw()
        want_q, want_s = orc.quant_act(xb)
        with_xsum = K % 64 == 0
        xq, sx, xsum = qk.qk_quantize_activations(to_dev_bf16(xb), with_xsum=with_xsum)
        assert np.array_equal(host(xq), want_q), (M, K)
        assert np.array_equal(host(sx).view(np.uint32), want_s.view(np.uint32)), (M, K)
        if with_xsum:
            assert np.array_equal(host(xsum), orc.group_sums(want_q)), (M, K)


def test_act_quant_golden_and_special_rows(qk, orc):
    from tests.test_oracle_pins import GOLDEN, bf16_bits

    with open(os.path.join(GOLDEN, "quant_act_rows.json")) as fh:
        rows = json.load(fh)["rows"]
    K = 64
    x = np.zeros((len(rows) + 3, K), np.float32)
    for i, r in enumerate(rows):
        x[i, : len(r["x"])] = r["x"]
    x[len(rows) + 0, 17] = -3.0                  # single nonzero
    x[len(rows) + 1, :] = 1e-30                  # tiny but in contract
    x[len(rows) + 2, ::2] = 65504.0              # large
    xb = bf16_bits(x)
    xq, sx, xsum = qk.qk_quantize_activations(to_dev_bf16(xb), with_xsum=True)
    for i, r in enumerate(rows):
        assert host(xq)[i, : len(r["codes"])].tolist() == r["codes"]
        assert float(host(sx)[i]) == r["scale"]
    want_q, want_s = orc.quant_act(xb)
    assert np.array_equal(host(xq), want_q)
    assert np.array_equal(host(sx), want_s)
    assert np.array_equal(host(xsum), orc.group_sums(want_q))


@pytest.mark.parametrize("case", [synthetic.DIT_ATTN, synthetic.DIT_MLP, *synthetic.SWEEP],
                         ids=lambda c: c.name)
def test_act_quant_full_configs(qk, orc, case):
    xb, _, _, _ = case.draw()
    want_q, want_s = orc.quant_act(xb)
    xq, sx, _ = qk.qk_quantize_activations(to_dev_bf16(xb))
    assert np.array_equal(host(xq), want_q)
    assert np.array_equal(host(sx), want_s)


@pytest.mark.parametrize("NK", [(128, 256), (3072, 3072), (48, 5120), (24, 32), (8, 65536)])
def test_w8_weight_quant_bit_exact(qk, orc, NK):
    N, K = NK
    rng = np.random.default_rng(N + K)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[N // 2] = 0.0
    Wq, sw = qk.qk_quantize_weights_int8(to_dev(W))
    want_q, want_s = orc.quant_w8(W)
    assert np.array_equal(host(Wq), want_q)
    assert np.array_equal(host(sw), want_s)


@pytest.mark.parametrize("NK", [(4096, 4096), (64, 64), (24, 320), (8, 65536)])
def test_w4_weight_quant_bit_exact(qk, orc, NK):
    N, K = NK
    rng = np.random.default_rng(N * 3 + K)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[0, 64:128] = 0.5                            # a constant group: scale 0
    Wp, s, o = qk.qk_quantize_weights_int4(to_dev(W))
    want_p, want_s, want_o = orc.quant_w4(W)
    assert np.array_equal(host(Wp), want_p)
    assert np.array_equal(t2bits(s), want_s)
    assert np.array_equal(t2bits(o), want_o)


def test_w4_golden_groups(qk):
    from tests.test_oracle_pins import unpack_codes, w4_golden_groups

    groups = w4_golden_groups()
    W = np.concatenate([g[0] for g in groups])[None, :]
    Wp, s, o = qk.qk_quantize_weights_int4(to_dev(W.astype(np.float32)))
    codes = unpack_codes(host(Wp))
    for i, (_, s16, o16, want) in enumerate(groups):
        assert t2bits(s)[0, i] == s16
        assert t2bits(o)[0, i] == o16
        assert codes[0, 64 * i: 64 * i + 64].tolist() == want
