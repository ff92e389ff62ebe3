"""Failure detection on the GPU without a fault: a kernel whose waits can never
complete gives up after its bound, records QK_ERR_TIMEOUT in the device error
word and returns; the host reads the status once, and the same context then
runs the real kernels normally."""
import pytest
import torch

from tests.gpu_common import qk  # noqa: F401

pytestmark = pytest.mark.gpu

QK_ERR_TIMEOUT = 7


def test_bounded_wait_reports_timeout_and_the_context_survives(qk):
    qk.qk_check_device_error()  # start clean
    qk.qk_debug_wait_timeout(2_000_000)  # about a millisecond per wait
    with pytest.raises(qk.QKError) as e:
        qk.qk_check_device_error()
    assert e.value.status == QK_ERR_TIMEOUT
    qk.qk_check_device_error()  # read once, then cleared
    # the context still runs the real path
    g = torch.Generator(device="cuda").manual_seed(0)
    x = torch.randn(64, 256, device="cuda", generator=g).to(torch.bfloat16)
    W = torch.randn(128, 256, device="cuda", generator=g) * 0.02
    Wq, sw = qk.qk_quantize_weights_int8(W)
    y = qk.qk_w8a8_linear(x, Wq, sw)
    torch.cuda.synchronize()
    qk.qk_check_device_error()
    xq, sx, _ = qk.qk_quantize_activations(x)
    ref = (xq.float() @ Wq.float().t()) * sx[:, None] * sw[None, :]
    assert torch.allclose(y.float(), ref, rtol=1e-2, atol=1e-2)


def test_timeout_on_another_stream_is_reported_there(qk):
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        qk.qk_debug_wait_timeout(1_000_000)
    with pytest.raises(qk.QKError) as e:
        qk.qk_check_device_error(stream=s)
    assert e.value.status == QK_ERR_TIMEOUT
    qk.qk_check_device_error()
