"""The C-ABI boundary on the CPU: the library loads without a GPU, exports every
function include/qk.h declares, and rejects bad arguments on the host with the
documented status codes before touching a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def qk():
    from w4a8_quantized_gemm_token_b200 import build

    build.build()
    from w4a8_quantized_gemm_token_b200 import binding

    return binding


def declared_functions():
    text = open(os.path.join(ROOT, "include", "qk.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qk_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_calls():
    names = declared_functions()
    for n in ("qk_quantize_weights_int8", "qk_quantize_weights_int4", "qk_quantize_activations",
              "qk_w8a8_linear", "qk_w4a8_linear", "qk_check_device_error", "qk_is_available"):
        assert n in names


def test_library_exports_every_declared_symbol(qk):
    for n in declared_functions():
        assert hasattr(qk.lib, n), n


def test_binding_types_every_declared_call(qk):
    """Every declared call has its argument and result types set in the binding
    (ctypes would otherwise pass 64-bit sizes as C ints)."""
    for n in declared_functions():
        assert n in qk._SIGS, n


def test_status_strings(qk):
    for s in range(8):
        assert qk.qk_status_string(s).startswith("QK_")
    assert "unknown" in qk.qk_status_string(99)


def test_workspace_sizes(qk):
    r = lambda b: (b + 255) // 256 * 256
    # codes, scales and one 8-byte readiness word per row (fused quantization)
    assert qk.qk_w8a8_workspace_size(16384, 3072) == r(16384 * 3072) + r(16384 * 4) + r(16384 * 8)
    assert qk.qk_w8a8_workspace_size(300, 64) == r(300 * 64) + r(300 * 4) + r(300 * 8)
    assert qk.qk_w4a8_workspace_size(17, 4096) == r(17 * 4096) + r(17 * 4) + r(17 * 64 * 4)
    assert qk.qk_w8a8_workspace_size(0, 256) == 0


FAKE = 1 << 20  # a 16-byte aligned, never dereferenced address


def call_w8a8(qk, x=FAKE, M=64, K=256, Wq=FAKE, sw=FAKE, bias=None, N=128, y=FAKE,
              ws=None, ws_bytes=0):
    return qk.lib.qk_w8a8_linear(x, M, K, Wq, sw, bias, N, y, ws, ws_bytes, None)


def test_shape_contract(qk):
    assert call_w8a8(qk, K=33) == 2
    assert call_w8a8(qk, K=16) == 2
    assert call_w8a8(qk, K=65536 + 32) == 2
    assert call_w8a8(qk, N=12) == 2
    assert call_w8a8(qk, N=0) == 2
    assert call_w8a8(qk, M=-1) == 1
    # W4A8 needs K % 64 == 0
    assert qk.lib.qk_w4a8_linear(FAKE, 8, 96, FAKE, FAKE, FAKE, None, 64, FAKE, None, 0, None) == 2


def test_empty_input_is_a_no_op(qk):
    assert call_w8a8(qk, M=0, x=None, y=None) == 0
    assert qk.lib.qk_quantize_activations(None, 0, 64, None, None, None, None) == 0


def test_null_and_misaligned_pointers(qk):
    assert call_w8a8(qk, x=None) == 1
    assert call_w8a8(qk, Wq=None) == 1
    assert call_w8a8(qk, y=FAKE + 8) == 3
    assert call_w8a8(qk, bias=FAKE + 4) == 3
    assert qk.lib.qk_quantize_activations(FAKE + 2, 4, 64, FAKE, FAKE, None, None) == 3


def test_routes_are_checked(qk):
    args = (FAKE, FAKE, FAKE, 32, 256, FAKE, FAKE, FAKE, None, 64, FAKE)
    assert qk.lib.qk_w4a8_gemm(*args, 2, None) == 1        # GEMV with M > 16
    assert qk.lib.qk_w4a8_gemm(*args, 7, None) == 1        # unknown route
    assert qk.lib.qk_w4a8_gemm(*args, 4, None) == 1
    # the plane-count hook: shape contract, null output, alignment
    assert qk.lib.qk_debug_w4a8_plane_count(FAKE, FAKE, 64, 96, ctypes.byref(ctypes.c_int()), None, None) == 2
    assert qk.lib.qk_debug_w4a8_plane_count(FAKE, FAKE, 64, 256, None, None, None) == 1
    assert qk.lib.qk_debug_w4a8_plane_count(FAKE + 2, FAKE, 64, 256, ctypes.byref(ctypes.c_int()), None, None) == 3
    assert qk.lib.qk_debug_w4a8_group_acc(FAKE, 8, 256, FAKE, 64, 4, 2, FAKE, 1, None) == 1
    # the timeout test hook checks its limit on the host
    assert qk.lib.qk_debug_wait_timeout(0, None) == 1
    assert qk.lib.qk_debug_wait_timeout((1 << 31) + 1, None) == 1


def test_no_device_here(qk):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert qk.qk_is_available(0) is False
    # valid arguments reach the device check and stop there, launching nothing
    assert call_w8a8(qk) == 4
    assert qk.lib.qk_quantize_weights_int8(FAKE, 128, 256, FAKE, FAKE, None) == 4
    assert qk.lib.qk_debug_wait_timeout(1000, None) == 4
    # every W4A8 GEMM route, the per-group fold included, stops at the device check
    for route in (0, 1, 3):
        assert qk.lib.qk_w4a8_gemm(FAKE, FAKE, FAKE, 32, 256, FAKE, FAKE, FAKE, None, 64, FAKE,
                                   route, None) == 4
    assert qk.lib.qk_debug_w4a8_plane_count(FAKE, FAKE, 64, 256, ctypes.byref(ctypes.c_int()), None, None) == 4


def test_binding_rejects_cpu_tensors(qk):
    import torch

    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        qk.qk_quantize_activations(x)
    with pytest.raises(TypeError):
        qk.qk_quantize_activations(x.float())


def test_w4a8_linear_plan(qk):
    """The routing query: one fused kernel for small M * K, quantization + GEMV
    for larger K at M <= 16, quantization + GEMM above M = 16."""
    assert qk.qk_w4a8_linear_plan(0, 64, 64) == qk.QK_PLAN_NONE
    assert qk.qk_w4a8_linear_plan(1, 4096, 4096) == qk.QK_PLAN_GEMV_QUANT
    assert qk.qk_w4a8_linear_plan(6, 4096, 4096) == qk.QK_PLAN_GEMV_QUANT
    assert qk.qk_w4a8_linear_plan(7, 4096, 4096) == qk.QK_PLAN_QUANT_GEMV
    assert qk.qk_w4a8_linear_plan(8, 4096, 4096) == qk.QK_PLAN_QUANT_GEMV
    assert qk.qk_w4a8_linear_plan(16, 4096, 4096) == qk.QK_PLAN_QUANT_GEMV
    assert qk.qk_w4a8_linear_plan(16, 3072, 128) == qk.QK_PLAN_QUANT_GEMV
    assert qk.qk_w4a8_linear_plan(12, 2112, 136) == qk.QK_PLAN_QUANT_GEMV
    # 65 groups: no GEMV tiling keeps a warp's groups in registers
    assert qk.qk_w4a8_linear_plan(16, 4160, 136) == qk.QK_PLAN_QUANT_GEMM
    assert qk.qk_w4a8_linear_plan(17, 4096, 4096) == qk.QK_PLAN_QUANT_GEMM
    assert qk.qk_w4a8_linear_plan(4, 32768, 64) == qk.QK_PLAN_QUANT_GEMM
    with pytest.raises(qk.QKError) as e:
        qk.qk_w4a8_linear_plan(8, 96, 64)  # K % 64 != 0
    assert e.value.status == 2


def test_prepared_w4a8_arguments(qk):
    """The prepared-weight calls: the size follows the route's scratch layout,
    and shapes, pointers, alignment (256 bytes for the prepared form) and the
    buffer size are checked on the host; valid arguments stop at the device
    check here."""
    import torch

    r = lambda b: (b + 255) // 256 * 256
    N, K = 264, 1024
    size = r(16) + r(N * 4) + r(N * 4) + r(-(-N // 60) * 8) + 3 * N * K
    assert qk.qk_w4a8_prepared_size(N, K) == size
    assert qk.qk_w4a8_prepared_size(N, 96) == 0        # K % 64 != 0
    assert qk.qk_w4a8_prepared_size(12, K) == 0        # N % 8 != 0
    planes = ctypes.byref(ctypes.c_int())
    prep = qk.lib.qk_w4a8_prepare
    assert prep(FAKE, FAKE, FAKE, N, 96, FAKE, size, planes, None) == 2
    assert prep(None, FAKE, FAKE, N, K, FAKE, size, planes, None) == 1
    assert prep(FAKE, FAKE, FAKE, N, K, None, size, planes, None) == 1
    assert prep(FAKE, FAKE, FAKE, N, K, FAKE + 16, size, planes, None) == 3
    assert prep(FAKE, FAKE + 2, FAKE, N, K, FAKE, size, planes, None) == 3
    assert prep(FAKE, FAKE, FAKE, N, K, FAKE, size - 1, planes, None) == 5
    gp = qk.lib.qk_w4a8_gemm_prepared
    assert gp(FAKE, FAKE, FAKE, 32, K, FAKE, FAKE, FAKE, None, None, N, FAKE, None) == 1
    assert gp(FAKE, FAKE, FAKE, 32, K, FAKE, FAKE, FAKE, FAKE + 16, None, N, FAKE, None) == 3
    assert gp(None, None, None, 0, K, None, None, None, None, None, N, None, None) == 0  # M = 0
    lp = qk.lib.qk_w4a8_linear_prepared
    assert lp(FAKE, 32, K, FAKE, FAKE, FAKE, None, None, N, FAKE, None, 0, None) == 1
    assert lp(FAKE, 32, K, FAKE, FAKE, FAKE, FAKE + 16, None, N, FAKE, None, 0, None) == 3
    assert lp(FAKE, 32, 96, FAKE, FAKE, FAKE, FAKE, None, N, FAKE, None, 0, None) == 2
    if not torch.cuda.is_available():
        assert prep(FAKE, FAKE, FAKE, N, K, FAKE, size, planes, None) == 4
        assert gp(FAKE, FAKE, FAKE, 32, K, FAKE, FAKE, FAKE, FAKE, None, N, FAKE, None) == 4
        assert lp(FAKE, 32, K, FAKE, FAKE, FAKE, FAKE, None, N, FAKE, None, 0, None) == 4
