"""Thin ctypes binding over libqk.so (include/qk.h), with the C names.

Argument marshalling only: each function checks tensor dtypes, devices and
contiguity, allocates outputs with ``torch.empty`` when the caller passes none,
and forwards raw device pointers plus the current torch stream to the C call.
Every step of the computation runs in the library's CUDA kernels; there is no
CPU fallback.  A non-zero status raises :class:`QKError`.  If the library has
not been built, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqk.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python -m w4a8_quantized_gemm_token_b200.build` "
        "(the quantized linear has no CPU fallback)")

lib = ctypes.CDLL(_LIB_PATH)

_P, _I64, _I, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "qk_status_string": (ctypes.c_char_p, [_I]),
    "qk_version": (_I, []),
    "qk_is_available": (_I, [_I]),
    "qk_w8a8_workspace_size": (_SZ, [_I64, _I64]),
    "qk_w4a8_workspace_size": (_SZ, [_I64, _I64]),
    "qk_quantize_weights_int8": (_I, [_P, _I64, _I64, _P, _P, _P]),
    "qk_quantize_weights_int4": (_I, [_P, _I64, _I64, _P, _P, _P, _P]),
    "qk_quantize_activations": (_I, [_P, _I64, _I64, _P, _P, _P, _P]),
    "qk_w8a8_linear": (_I, [_P, _I64, _I64, _P, _P, _P, _I64, _P, _P, _SZ, _P]),
    "qk_w8a8_linear_fused": (_I, [_P, _I64, _I64, _P, _P, _P, _I64, _P, _P, _SZ, _P]),
    "qk_w8a8_gemm": (_I, [_P, _P, _I64, _I64, _P, _P, _P, _I64, _P, _P]),
    "qk_w8a8_linear_gated": (_I, [_P, _I64, _I64, _P, _P, _P, _P, _P, _I64, _P, _P, _SZ, _P]),
    "qk_w8a8_linear_noalloc": (_I, [_P, _I64, _I64, _P, _P, _P, _I64, _P, _P]),
    "qk_w4a8_linear": (_I, [_P, _I64, _I64, _P, _P, _P, _P, _I64, _P, _P, _SZ, _P]),
    "qk_w4a8_gemm": (_I, [_P, _P, _P, _I64, _I64, _P, _P, _P, _P, _I64, _P, _I, _P]),
    "qk_w4a8_linear_plan": (_I, [_I64, _I64, _I64]),
    "qk_w4a8_prepared_size": (_SZ, [_I64, _I64]),
    "qk_w4a8_prepare": (_I, [_P, _P, _P, _I64, _I64, _P, _SZ, _P, _P]),
    "qk_w4a8_gemm_prepared": (_I, [_P, _P, _P, _I64, _I64, _P, _P, _P, _P, _P, _I64, _P, _P]),
    "qk_w4a8_linear_prepared": (_I, [_P, _I64, _I64, _P, _P, _P, _P, _P, _I64, _P, _P, _SZ,
                                     _P]),
    "qk_check_device_error": (_I, [_P]),
    "qk_debug_w8a8_acc": (_I, [_P, _I64, _I64, _P, _I64, _P, _P]),
    "qk_debug_w4a8_group_acc": (_I, [_P, _I64, _I64, _P, _I64, _I64, _I64, _P, _I, _P]),
    "qk_debug_wait_timeout": (_I, [_I64, _P]),
    "qk_debug_int8_peak": (_I, [_I64, _P, _P]),
    "qk_debug_w4a8_plane_count": (_I, [_P, _P, _I64, _I64, _P, _P, _P]),
    "qk_sage_attention_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "qk_sage_attention": (_I, [_P, _P, _P, _I64, _I64, _I64, _I64, ctypes.c_float, _P, _P, _SZ, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

QK_OK = 0
QK_ROUTE_AUTO, QK_ROUTE_GEMM, QK_ROUTE_GEMV, QK_ROUTE_GEMM_FOLD = 0, 1, 2, 3
QK_PLAN_NONE, QK_PLAN_GEMV_QUANT, QK_PLAN_QUANT_GEMV, QK_PLAN_QUANT_GEMM = 0, 1, 2, 3


class QKError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {qk_status_string(status)}")


def qk_status_string(status: int) -> str:
    return lib.qk_status_string(status).decode()


def qk_version() -> int:
    return lib.qk_version()


def qk_is_available(device: int = 0) -> bool:
    return bool(lib.qk_is_available(device))


def qk_w4a8_linear_plan(M: int, K: int, N: int) -> int:
    """The kernels qk_w4a8_linear launches for this shape (a QK_PLAN_* value);
    raises QKError for an invalid shape."""
    r = lib.qk_w4a8_linear_plan(M, K, N)
    if r < 0:
        raise QKError(-r, "qk_w4a8_linear_plan")
    return r


def qk_w8a8_workspace_size(M: int, K: int) -> int:
    return lib.qk_w8a8_workspace_size(M, K)


def qk_w4a8_workspace_size(M: int, K: int) -> int:
    return lib.qk_w4a8_workspace_size(M, K)


# ------------------------------------------------------------- marshalling

def _check(status: int, where: str) -> None:
    if status != QK_OK:
        raise QKError(status, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _need(t, dtype, ndim, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _out(t, shape, dtype, device, name):
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    _need(t, dtype, len(shape), name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


# --------------------------------------------------------------- the calls

def qk_quantize_weights_int8(W, Wq=None, sw=None, stream=None):
    """W fp32 [N, K] -> (Wq int8 [N, K], sw fp32 [N])."""
    _need(W, torch.float32, 2, "W")
    N, K = W.shape
    Wq = _out(Wq, (N, K), torch.int8, W.device, "Wq")
    sw = _out(sw, (N,), torch.float32, W.device, "sw")
    _check(lib.qk_quantize_weights_int8(_ptr(W), N, K, _ptr(Wq), _ptr(sw), _stream(stream)),
           "qk_quantize_weights_int8")
    return Wq, sw


def qk_quantize_weights_int4(W, Wp=None, wscale=None, woffset=None, stream=None):
    """W fp32 [N, K] -> (Wp uint8 [N, K/2], wscale fp16 [N, K/64], woffset fp16 [N, K/64])."""
    _need(W, torch.float32, 2, "W")
    N, K = W.shape
    Wp = _out(Wp, (N, K // 2), torch.uint8, W.device, "Wp")
    wscale = _out(wscale, (N, K // 64), torch.float16, W.device, "wscale")
    woffset = _out(woffset, (N, K // 64), torch.float16, W.device, "woffset")
    _check(lib.qk_quantize_weights_int4(_ptr(W), N, K, _ptr(Wp), _ptr(wscale), _ptr(woffset),
                                        _stream(stream)), "qk_quantize_weights_int4")
    return Wp, wscale, woffset


def qk_quantize_activations(x, xq=None, sx=None, xsum=None, with_xsum=False, stream=None):
    """x bf16 [M, K] -> (xq int8 [M, K], sx fp32 [M], xsum int32 [M, K/64] or None)."""
    _need(x, torch.bfloat16, 2, "x")
    M, K = x.shape
    xq = _out(xq, (M, K), torch.int8, x.device, "xq")
    sx = _out(sx, (M,), torch.float32, x.device, "sx")
    if with_xsum or xsum is not None:
        xsum = _out(xsum, (M, K // 64), torch.int32, x.device, "xsum")
    _check(lib.qk_quantize_activations(_ptr(x), M, K, _ptr(xq), _ptr(sx), _ptr(xsum),
                                       _stream(stream)), "qk_quantize_activations")
    return xq, sx, xsum


def qk_w8a8_linear(x, Wq, sw, bias=None, y=None, workspace=None, stream=None, fused=False):
    """y bf16 [M, N] = bf16(quant(x) . Wq^T * sx * sw + bias).  fused=True calls
    qk_w8a8_linear_fused (the same result from one kernel)."""
    _need(x, torch.bfloat16, 2, "x")
    _need(Wq, torch.int8, 2, "Wq")
    _need(sw, torch.float32, 1, "sw")
    if bias is not None:
        _need(bias, torch.float32, 1, "bias")
    M, K = x.shape
    N = Wq.shape[0]
    y = _out(y, (M, N), torch.bfloat16, x.device, "y")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    fn = lib.qk_w8a8_linear_fused if fused else lib.qk_w8a8_linear
    _check(fn(_ptr(x), M, K, _ptr(Wq), _ptr(sw), _ptr(bias), N, _ptr(y), _ptr(workspace),
              ws_bytes, _stream(stream)), "qk_w8a8_linear_fused" if fused else "qk_w8a8_linear")
    return y


def qk_w8a8_linear_gated(x, Wq, sw, bias, gate, residual, y=None, workspace=None, stream=None):
    """y bf16 [M, N] = bf16(residual + gate * (quant(x) . Wq^T * sx * sw + bias));
    y may be `residual` itself (an in-place update)."""
    _need(x, torch.bfloat16, 2, "x")
    _need(Wq, torch.int8, 2, "Wq")
    _need(sw, torch.float32, 1, "sw")
    _need(gate, torch.float32, 1, "gate")
    _need(residual, torch.bfloat16, 2, "residual")
    if bias is not None:
        _need(bias, torch.float32, 1, "bias")
    M, K = x.shape
    N = Wq.shape[0]
    if tuple(residual.shape) != (M, N) or gate.shape[0] != N:
        raise ValueError("residual must be [M, N] and gate [N]")
    y = _out(y, (M, N), torch.bfloat16, x.device, "y")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.qk_w8a8_linear_gated(_ptr(x), M, K, _ptr(Wq), _ptr(sw), _ptr(bias), _ptr(gate),
                                    _ptr(residual), N, _ptr(y), _ptr(workspace), ws_bytes,
                                    _stream(stream)), "qk_w8a8_linear_gated")
    return y


def qk_w8a8_gemm(xq, sx, Wq, sw, bias=None, y=None, stream=None):
    _need(xq, torch.int8, 2, "xq")
    _need(sx, torch.float32, 1, "sx")
    _need(Wq, torch.int8, 2, "Wq")
    _need(sw, torch.float32, 1, "sw")
    if bias is not None:
        _need(bias, torch.float32, 1, "bias")
    M, K = xq.shape
    N = Wq.shape[0]
    y = _out(y, (M, N), torch.bfloat16, xq.device, "y")
    _check(lib.qk_w8a8_gemm(_ptr(xq), _ptr(sx), M, K, _ptr(Wq), _ptr(sw), _ptr(bias), N, _ptr(y),
                            _stream(stream)), "qk_w8a8_gemm")
    return y


def qk_w8a8_linear_noalloc(x, Wq, sw, bias=None, y=None, stream=None):
    """The W8A8 linear on the library's per-device scratch (no allocation per
    call; calls must not overlap on the device, see include/qk.h)."""
    _need(x, torch.bfloat16, 2, "x")
    _need(Wq, torch.int8, 2, "Wq")
    _need(sw, torch.float32, 1, "sw")
    if bias is not None:
        _need(bias, torch.float32, 1, "bias")
    M, K = x.shape
    N = Wq.shape[0]
    y = _out(y, (M, N), torch.bfloat16, x.device, "y")
    _check(lib.qk_w8a8_linear_noalloc(_ptr(x), M, K, _ptr(Wq), _ptr(sw), _ptr(bias), N, _ptr(y),
                                      _stream(stream)),
           "qk_w8a8_linear_noalloc")
    return y


def qk_w4a8_linear(x, Wp, wscale, woffset, bias=None, y=None, workspace=None, stream=None):
    _need(x, torch.bfloat16, 2, "x")
    _need(Wp, torch.uint8, 2, "Wp")
    _need(wscale, torch.float16, 2, "wscale")
    _need(woffset, torch.float16, 2, "woffset")
    if bias is not None:
        _need(bias, torch.float32, 1, "bias")
    M, K = x.shape
    N = Wp.shape[0]
    y = _out(y, (M, N), torch.bfloat16, x.device, "y")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.qk_w4a8_linear(_ptr(x), M, K, _ptr(Wp), _ptr(wscale), _ptr(woffset), _ptr(bias),
                              N, _ptr(y), _ptr(workspace), ws_bytes, _stream(stream)),
           "qk_w4a8_linear")
    return y


def qk_w4a8_prepared_size(N: int, K: int) -> int:
    return int(lib.qk_w4a8_prepared_size(int(N), int(K)))


def qk_w4a8_prepare(Wp, wscale, woffset, prepared=None, stream=None):
    """(prepared uint8 tensor, plane count): the GEMM route's digit planes of
    the weight, built once for the _prepared calls (plane count 1..3, or 255
    when the per-group fold computes the product)."""
    _need(Wp, torch.uint8, 2, "Wp")
    _need(wscale, torch.float16, 2, "wscale")
    _need(woffset, torch.float16, 2, "woffset")
    N, K = Wp.shape[0], Wp.shape[1] * 2
    if prepared is None:
        size = lib.qk_w4a8_prepared_size(N, K)
        prepared = torch.empty(max(int(size), 1), dtype=torch.uint8, device=Wp.device)
    else:
        _need(prepared, torch.uint8, 1, "prepared")
    planes = ctypes.c_int(0)
    _check(lib.qk_w4a8_prepare(_ptr(Wp), _ptr(wscale), _ptr(woffset), N, K, _ptr(prepared),
                               prepared.numel(), ctypes.byref(planes), _stream(stream)),
           "qk_w4a8_prepare")
    return prepared, int(planes.value)


def qk_w4a8_linear_prepared(x, Wp, wscale, woffset, prepared, bias=None, y=None, workspace=None,
                            stream=None):
    _need(x, torch.bfloat16, 2, "x")
    _need(Wp, torch.uint8, 2, "Wp")
    _need(wscale, torch.float16, 2, "wscale")
    _need(woffset, torch.float16, 2, "woffset")
    _need(prepared, torch.uint8, 1, "prepared")
    if bias is not None:
        _need(bias, torch.float32, 1, "bias")
    M, K = x.shape
    N = Wp.shape[0]
    y = _out(y, (M, N), torch.bfloat16, x.device, "y")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.qk_w4a8_linear_prepared(_ptr(x), M, K, _ptr(Wp), _ptr(wscale), _ptr(woffset),
                                       _ptr(prepared), _ptr(bias), N, _ptr(y), _ptr(workspace),
                                       ws_bytes, _stream(stream)),
           "qk_w4a8_linear_prepared")
    return y


def qk_w4a8_gemm_prepared(xq, sx, xsum, Wp, wscale, woffset, prepared, bias=None, y=None,
                          stream=None):
    _need(xq, torch.int8, 2, "xq")
    _need(sx, torch.float32, 1, "sx")
    _need(xsum, torch.int32, 2, "xsum")
    _need(Wp, torch.uint8, 2, "Wp")
    _need(wscale, torch.float16, 2, "wscale")
    _need(woffset, torch.float16, 2, "woffset")
    _need(prepared, torch.uint8, 1, "prepared")
    if bias is not None:
        _need(bias, torch.float32, 1, "bias")
    M, K = xq.shape
    N = Wp.shape[0]
    y = _out(y, (M, N), torch.bfloat16, xq.device, "y")
    _check(lib.qk_w4a8_gemm_prepared(_ptr(xq), _ptr(sx), _ptr(xsum), M, K, _ptr(Wp),
                                     _ptr(wscale), _ptr(woffset), _ptr(prepared), _ptr(bias), N,
                                     _ptr(y), _stream(stream)),
           "qk_w4a8_gemm_prepared")
    return y


def qk_w4a8_gemm(xq, sx, xsum, Wp, wscale, woffset, bias=None, y=None, route=QK_ROUTE_AUTO,
                 stream=None):
    _need(xq, torch.int8, 2, "xq")
    _need(sx, torch.float32, 1, "sx")
    _need(xsum, torch.int32, 2, "xsum")
    _need(Wp, torch.uint8, 2, "Wp")
    _need(wscale, torch.float16, 2, "wscale")
    _need(woffset, torch.float16, 2, "woffset")
    if bias is not None:
        _need(bias, torch.float32, 1, "bias")
    M, K = xq.shape
    N = Wp.shape[0]
    y = _out(y, (M, N), torch.bfloat16, xq.device, "y")
    _check(lib.qk_w4a8_gemm(_ptr(xq), _ptr(sx), _ptr(xsum), M, K, _ptr(Wp), _ptr(wscale),
                            _ptr(woffset), _ptr(bias), N, _ptr(y), int(route), _stream(stream)),
           "qk_w4a8_gemm")
    return y


def qk_check_device_error(stream=None) -> None:
    _check(lib.qk_check_device_error(_stream(stream)), "qk_check_device_error")


def qk_debug_w8a8_acc(xq, Wq, acc=None, stream=None):
    _need(xq, torch.int8, 2, "xq")
    _need(Wq, torch.int8, 2, "Wq")
    M, K = xq.shape
    N = Wq.shape[0]
    acc = _out(acc, (M, N), torch.int32, xq.device, "acc")
    _check(lib.qk_debug_w8a8_acc(_ptr(xq), M, K, _ptr(Wq), N, _ptr(acc), _stream(stream)),
           "qk_debug_w8a8_acc")
    return acc


def qk_debug_w4a8_group_acc(xq, Wp, m0, m1, route, acc=None, stream=None):
    _need(xq, torch.int8, 2, "xq")
    _need(Wp, torch.uint8, 2, "Wp")
    M, K = xq.shape
    N = Wp.shape[0]
    acc = _out(acc, (m1 - m0, N, K // 64), torch.int32, xq.device, "acc")
    _check(lib.qk_debug_w4a8_group_acc(_ptr(xq), M, K, _ptr(Wp), N, m0, m1, _ptr(acc), int(route),
                                       _stream(stream)), "qk_debug_w4a8_group_acc")
    return acc


def qk_debug_w4a8_plane_count(wscale, woffset, K: int, stream=None, with_mixed=False):
    """Digit planes the W4A8 GEMM route needs for these scales and offsets
    (1..3), or 255 when it takes the per-group fold kernel; with
    `with_mixed`, also whether a three-plane weight takes the mixed layout."""
    _need(wscale, torch.float16, 2, "wscale")
    _need(woffset, torch.float16, 2, "woffset")
    N = wscale.shape[0]
    planes = ctypes.c_int(0)
    mixed = ctypes.c_int(0)
    _check(lib.qk_debug_w4a8_plane_count(_ptr(wscale), _ptr(woffset), N, int(K),
                                         ctypes.byref(planes), ctypes.byref(mixed),
                                         _stream(stream)),
           "qk_debug_w4a8_plane_count")
    return (int(planes.value), bool(mixed.value)) if with_mixed else int(planes.value)


def qk_debug_wait_timeout(limit_cycles: int, stream=None) -> None:
    """Launch the test kernel whose waits can never complete; each gives up
    after `limit_cycles` SM cycles and records QK_ERR_TIMEOUT for
    qk_check_device_error."""
    _check(lib.qk_debug_wait_timeout(int(limit_cycles), _stream(stream)), "qk_debug_wait_timeout")


def qk_debug_int8_peak(iters: int, stream=None) -> float:
    """Launch the INT8 tensor-pipe probe (`iters` x 8 kind::i8 MMAs of
    256 x 256 x 32 per CTA pair); returns the int8 operations it performs."""
    ops = ctypes.c_double(0.0)
    _check(lib.qk_debug_int8_peak(int(iters), ctypes.byref(ops), _stream(stream)),
           "qk_debug_int8_peak")
    return float(ops.value)


def qk_sage_attention_workspace_size(B: int, H: int, L: int) -> int:
    return int(lib.qk_sage_attention_workspace_size(B, H, L))


def qk_sage_attention(q, k, v, scale=None, out=None, workspace=None, stream=None):
    """INT8 attention over bf16 [B, H, L, 128] q, k, v; returns bf16 [B, H, L, 128]."""
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, 4, name)
    B, H, L, D = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k and v must have the same shape [B, H, L, 128]")
    out = _out(out, (B, H, L, D), torch.bfloat16, q.device, "out")
    if scale is None:
        scale = D ** -0.5
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.qk_sage_attention(_ptr(q), _ptr(k), _ptr(v), B, H, L, D, float(scale), _ptr(out),
                                 _ptr(workspace), ws_bytes, _stream(stream)), "qk_sage_attention")
    return out
