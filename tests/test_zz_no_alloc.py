"""qk_w8a8_linear_noalloc, the W8A8 linear for callers that cannot allocate
device memory (a custom allocator owns it all, a fixed-budget real-time host,
a plugin whose host forbids allocation in callbacks).  It keeps its scratch in a
64 MiB array built into the library instead of a workspace.

Called through the C ABI; each of two calls in a row (different shapes, so the
second runs over what the first left in the shared scratch) must match the
regular qk_w8a8_linear within the 2-ulp tolerance of the other tests.  This file
sorts last so that a run stopping at the first failure has run everything else."""
import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_common import qk, t2bits, to_dev, to_dev_bf16  # noqa: F401
from tests.helpers import bf16_ulp_distance
from w4a8_quantized_gemm_token_b200 import synthetic

pytestmark = pytest.mark.gpu

TOL_ULP = 2
SCRATCH_BYTES = 64 * 1024 * 1024
QK_ERR_WORKSPACE = 5


def noalloc_fn(qk):
    fn = qk.lib.qk_w8a8_linear_noalloc
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    fn.restype = ctypes.c_int
    fn.argtypes = [P, I64, I64, P, P, P, I64, P, P]
    return fn


def call_noalloc(fn, x, Wq, sw, bias, y):
    M, K = x.shape
    N = Wq.shape[0]
    return fn(x.data_ptr(), M, K, Wq.data_ptr(), sw.data_ptr(),
              None if bias is None else bias.data_ptr(), N, y.data_ptr(),
              torch.cuda.current_stream().cuda_stream)


def make(qk, case):
    xb, W, b, _ = case.draw()
    Wq, sw = qk.qk_quantize_weights_int8(to_dev(W))
    return to_dev_bf16(xb), Wq, sw, (to_dev(b) if b is not None else None)


def test_noalloc_matches_linear_on_two_calls_in_a_row(qk):
    fn = noalloc_fn(qk)
    cases = [synthetic.LinearCase("na1", M=777, K=3072, N=1032, outlier_frac=0.01, seed=21),
             synthetic.LinearCase("na2", M=130, K=512, N=264, bias=False, seed=22)]
    prepared = [make(qk, c) for c in cases]
    outs = []
    for x, Wq, sw, bias in prepared:                      # two calls in a row
        y = torch.empty(x.shape[0], Wq.shape[0], dtype=torch.bfloat16, device="cuda")
        assert call_noalloc(fn, x, Wq, sw, bias, y) == 0
        outs.append(y)
    torch.cuda.synchronize()
    qk.qk_check_device_error()
    for (x, Wq, sw, bias), y in zip(prepared, outs):
        ref = qk.qk_w8a8_linear(x, Wq, sw, bias)
        torch.cuda.synchronize()
        d = bf16_ulp_distance(t2bits(y), t2bits(ref))
        assert d.max() <= TOL_ULP, f"worst {d.max()} ulp"


def test_noalloc_allocates_nothing_after_its_first_call(qk):
    fn = noalloc_fn(qk)
    x, Wq, sw, bias = make(qk, synthetic.LinearCase("na3", M=512, K=1024, N=512, seed=23))
    y = torch.empty(512, 512, dtype=torch.bfloat16, device="cuda")
    assert call_noalloc(fn, x, Wq, sw, bias, y) == 0      # loads the module if needed
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert call_noalloc(fn, x, Wq, sw, bias, y) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_rejects_problems_beyond_its_scratch(qk):
    fn = noalloc_fn(qk)
    K = 4096
    M = SCRATCH_BYTES // K + 1                            # codes alone exceed the scratch
    assert qk.qk_w8a8_workspace_size(M, K) > SCRATCH_BYTES
    x = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros(64, K, dtype=torch.int8, device="cuda")
    sw = torch.ones(64, dtype=torch.float32, device="cuda")
    y = torch.full((M, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    assert call_noalloc(fn, x, Wq, sw, None, y) == QK_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())                         # nothing was launched
