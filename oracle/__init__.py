"""CPU oracle for the W8A8 / W4A8 quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library never calls it, and this package imports nothing
from the library.  The arithmetic lives in ``qk_oracle.c`` (plain C, built
strictly with gcc); this module only marshals numpy arrays to it.

Every function takes and returns numpy arrays.  bf16 and fp16 values travel as
their uint16 bit patterns.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qk_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile ``qk_oracle.c`` into ``liboracle.so`` next to it (gcc, strict fp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _bind(path: str):
    lib = ctypes.CDLL(path)
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    sigs = {
        "oracle_bf16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
        "oracle_f32_to_f16": (ctypes.c_uint16, [ctypes.c_float]),
        "oracle_f16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
        "oracle_f64_to_bf16": (ctypes.c_uint16, [ctypes.c_double]),
        "oracle_set_threads": (ctypes.c_int, [ctypes.c_int]),
        "oracle_quant_act_bf16": (None, [P, I64, I64, P, P]),
        "oracle_quant_w8": (None, [P, I64, I64, P, P]),
        "oracle_group_sums": (None, [P, I64, I64, P]),
        "oracle_quant_w4": (None, [P, I64, I64, P, P, P]),
        "oracle_w8a8_acc": (None, [P, I64, I64, P, I64, P]),
        "oracle_w4a8_group_acc": (None, [P, I64, I64, P, I64, P]),
        "oracle_w8a8_dequant": (None, [P, I64, I64, P, P, P, P]),
        "oracle_w8a8_gated": (None, [P, I64, I64, P, P, P, P, P, P]),
        "oracle_w4a8_dequant": (None, [P, P, I64, I64, I64, P, P, P, P, P]),
        "oracle_w8a8_dequant_f64": (None, [P, I64, I64, P, P, P, P]),
        "oracle_w4a8_dequant_f64": (None, [P, P, I64, I64, I64, P, P, P, P, P]),
        "oracle_sage_attention": (None, [P, P, P, P, P, I64, I64, ctypes.c_double, P, P]),
        "oracle_sage_attention_rows": (None, [P, P, P, P, P, I64, I64, ctypes.c_double, P, I64,
                                              P, P]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build())
        _lib.oracle_set_threads(int(os.environ.get("QK_ORACLE_THREADS", "1")))
    return _lib


def set_threads(n: int) -> int:
    """Let the oracle's row loops use `n` OpenMP threads (each output is still
    computed by one thread in the same order, so results do not change);
    returns the count in effect."""
    return int(_load().oracle_set_threads(int(n)))


@contextlib.contextmanager
def using_library(path: str):
    """Temporarily route every oracle call to another build of ``qk_oracle.c``
    (the mutation test plants mistakes in a copy and checks that the pins fail)."""
    global _lib
    saved = _load()
    _lib = _bind(path)
    _lib.oracle_set_threads(int(os.environ.get("QK_ORACLE_THREADS", "1")))
    try:
        yield
    finally:
        _lib = saved


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _p(a):
    return None if a is None else a.ctypes.data


# ------------------------------------------------------------------ scalars

def f64_to_bf16(v: float) -> int:
    return int(_load().oracle_f64_to_bf16(float(v)))


def f32_to_f16(v: float) -> int:
    return int(_load().oracle_f32_to_f16(float(v)))


def f16_to_f32(u: int) -> float:
    return float(_load().oracle_f16_to_f32(int(u)))


def f64_to_bf16_array(v: np.ndarray) -> np.ndarray:
    f = _load().oracle_f64_to_bf16
    flat = np.asarray(v, dtype=np.float64).ravel()
    return np.array([f(float(t)) for t in flat], dtype=np.uint16).reshape(np.shape(v))


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------------- quant

def quant_act(x_bf16: np.ndarray):
    """x bf16 bits [M, K] -> (xq int8 [M, K], sx float32 [M])."""
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    xq = np.empty((M, K), np.int8)
    sx = np.empty(M, np.float32)
    _load().oracle_quant_act_bf16(_p(x), M, K, _p(xq), _p(sx))
    return xq, sx


def quant_w8(W: np.ndarray):
    """W float32 [N, K] -> (Wq int8 [N, K], sw float32 [N])."""
    W = _c(W, np.float32)
    N, K = W.shape
    Wq = np.empty((N, K), np.int8)
    sw = np.empty(N, np.float32)
    _load().oracle_quant_w8(_p(W), N, K, _p(Wq), _p(sw))
    return Wq, sw


def group_sums(xq: np.ndarray) -> np.ndarray:
    """xq int8 [M, K] -> xsum int32 [M, K/64]."""
    xq = _c(xq, np.int8)
    M, K = xq.shape
    assert K % 64 == 0
    out = np.empty((M, K // 64), np.int32)
    _load().oracle_group_sums(_p(xq), M, K, _p(out))
    return out


def quant_w4(W: np.ndarray):
    """W float32 [N, K] -> (Wp uint8 [N, K/2], s fp16 bits [N, K/64], o fp16 bits [N, K/64])."""
    W = _c(W, np.float32)
    N, K = W.shape
    assert K % 64 == 0
    Wp = np.empty((N, K // 2), np.uint8)
    s = np.empty((N, K // 64), np.uint16)
    o = np.empty((N, K // 64), np.uint16)
    _load().oracle_quant_w4(_p(W), N, K, _p(Wp), _p(s), _p(o))
    return Wp, s, o


# -------------------------------------------------------------- accumulate

def w8a8_acc(xq: np.ndarray, Wq: np.ndarray) -> np.ndarray:
    """Exact int64 acc [M, N] = xq [M, K] . Wq [N, K]^T."""
    xq = _c(xq, np.int8)
    Wq = _c(Wq, np.int8)
    M, K = xq.shape
    N = Wq.shape[0]
    assert Wq.shape[1] == K
    acc = np.empty((M, N), np.int64)
    _load().oracle_w8a8_acc(_p(xq), M, K, _p(Wq), N, _p(acc))
    return acc


def w4a8_group_acc(xq: np.ndarray, Wp: np.ndarray) -> np.ndarray:
    """Exact int64 per-group acc [M, N, K/64] on the raw codes 0..15."""
    xq = _c(xq, np.int8)
    Wp = _c(Wp, np.uint8)
    M, K = xq.shape
    N = Wp.shape[0]
    assert Wp.shape[1] * 2 == K and K % 64 == 0
    acc = np.empty((M, N, K // 64), np.int64)
    _load().oracle_w4a8_group_acc(_p(xq), M, K, _p(Wp), N, _p(acc))
    return acc


# ----------------------------------------------------------------- dequant

def w8a8_dequant(acc, sx, sw, bias=None) -> np.ndarray:
    """bf16 bits [M, N] of acc * sx * sw + bias evaluated in fp64, rounded once."""
    acc = _c(acc, np.int64)
    M, N = acc.shape
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    y = np.empty((M, N), np.uint16)
    _load().oracle_w8a8_dequant(_p(acc), M, N, _p(sx), _p(sw), _p(b), _p(y))
    return y


def w8a8_gated(acc, sx, sw, bias, gate, r_bf16) -> np.ndarray:
    """bf16 bits [M, N] of r + gate * (acc * sx * sw + bias) in fp64, rounded once."""
    acc = _c(acc, np.int64)
    M, N = acc.shape
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    g = _c(gate, np.float32)
    r = _c(r_bf16, np.uint16)
    assert g.shape == (N,) and r.shape == (M, N)
    out = np.empty((M, N), np.uint16)
    _load().oracle_w8a8_gated(_p(acc), M, N, _p(sx), _p(sw), _p(b), _p(g), _p(r), _p(out))
    return out


def w8a8_dequant_f64(acc, sx, sw, bias=None) -> np.ndarray:
    """fp64 value [M, N] of acc * sx * sw + bias, before the bf16 rounding."""
    acc = _c(acc, np.int64)
    M, N = acc.shape
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    v = np.empty((M, N), np.float64)
    _load().oracle_w8a8_dequant_f64(_p(acc), M, N, _p(sx), _p(sw), _p(b), _p(v))
    return v


def w4a8_dequant_f64(acc_g, xsum, sx, s16, o16, bias=None) -> np.ndarray:
    """fp64 value [M, N] of sx * sum_g(s * acc_g + o * xsum_g) + bias, before rounding."""
    acc_g = _c(acc_g, np.int64)
    M, N, G = acc_g.shape
    xsum = _c(xsum, np.int32)
    sx = _c(sx, np.float32)
    s16 = _c(s16, np.uint16)
    o16 = _c(o16, np.uint16)
    b = None if bias is None else _c(bias, np.float32)
    v = np.empty((M, N), np.float64)
    _load().oracle_w4a8_dequant_f64(_p(acc_g), _p(xsum), M, N, G, _p(sx), _p(s16), _p(o16),
                                    _p(b), _p(v))
    return v


def w4a8_dequant(acc_g, xsum, sx, s16, o16, bias=None) -> np.ndarray:
    """bf16 bits [M, N] of sx * sum_g(s * acc_g + o * xsum_g) + bias in fp64."""
    acc_g = _c(acc_g, np.int64)
    M, N, G = acc_g.shape
    xsum = _c(xsum, np.int32)
    sx = _c(sx, np.float32)
    s16 = _c(s16, np.uint16)
    o16 = _c(o16, np.uint16)
    b = None if bias is None else _c(bias, np.float32)
    y = np.empty((M, N), np.uint16)
    _load().oracle_w4a8_dequant(_p(acc_g), _p(xsum), M, N, G, _p(sx), _p(s16), _p(o16),
                                _p(b), _p(y))
    return y


# ------------------------------------------------------------ whole linear

def w8a8_linear(x_bf16, Wq, sw, bias=None):
    """The W8A8 linear on bf16 rows: returns (y bf16 bits, xq, sx, acc)."""
    xq, sx = quant_act(x_bf16)
    acc = w8a8_acc(xq, Wq)
    return w8a8_dequant(acc, sx, sw, bias), xq, sx, acc


def w8a8_linear_gated(x_bf16, Wq, sw, bias, gate, r_bf16):
    """The W8A8 linear with the gated residual epilogue: (out bf16 bits, xq, sx, acc)."""
    xq, sx = quant_act(x_bf16)
    acc = w8a8_acc(xq, Wq)
    return w8a8_gated(acc, sx, sw, bias, gate, r_bf16), xq, sx, acc


def w4a8_linear(x_bf16, Wp, s16, o16, bias=None):
    """The W4A8 linear on bf16 rows: returns (y bf16 bits, xq, sx, xsum, acc_g)."""
    xq, sx = quant_act(x_bf16)
    xsum = group_sums(xq)
    acc_g = w4a8_group_acc(xq, Wp)
    return w4a8_dequant(acc_g, xsum, sx, s16, o16, bias), xq, sx, xsum, acc_g


def sage_attention_head(q_bf16, k_bf16, v_bf16, scale, with_f64=False):
    """INT8 attention of one head ("qlip-mlx" README, "sage_attention"; R14):
    q, k, v bf16 bits [L, D].  q and k are quantized per token (quant_act),
    scores and softmax and P V in fp64, the output rounded once to bf16.
    Returns bf16 bits [L, D] (and the fp64 output when `with_f64`)."""
    q = _c(q_bf16, np.uint16)
    k = _c(k_bf16, np.uint16)
    v = _c(v_bf16, np.uint16)
    L, D = q.shape
    assert k.shape == (L, D) and v.shape == (L, D)
    qc, sq = quant_act(q)
    kc, sk = quant_act(k)
    out = np.empty((L, D), np.uint16)
    o64 = np.empty((L, D), np.float64) if with_f64 else None
    _load().oracle_sage_attention(_p(qc), _p(sq), _p(kc), _p(sk), _p(v), L, D, float(scale),
                                  _p(o64) if with_f64 else None, _p(out))
    return (out, o64) if with_f64 else out


def sage_attention_rows(q_bf16, k_bf16, v_bf16, scale, rows):
    """sage_attention_head for the query rows `rows` only: (bf16 bits, fp64)
    outputs [len(rows), D] (same arithmetic, for sampled rows of long heads)."""
    q = _c(q_bf16, np.uint16)
    k = _c(k_bf16, np.uint16)
    v = _c(v_bf16, np.uint16)
    L, D = q.shape
    rows = _c(np.asarray(rows), np.int64)
    qc, sq = quant_act(q)
    kc, sk = quant_act(k)
    out = np.empty((len(rows), D), np.uint16)
    o64 = np.empty((len(rows), D), np.float64)
    _load().oracle_sage_attention_rows(_p(qc), _p(sq), _p(kc), _p(sk), _p(v), L, D, float(scale),
                                       _p(rows), len(rows), _p(o64), _p(out))
    return out, o64


def sage_attention(q_bf16, k_bf16, v_bf16, scale, with_f64=False):
    """sage_attention_head over [B, H, L, D] bf16 bits, head by head."""
    B, H, L, D = q_bf16.shape
    out = np.empty((B, H, L, D), np.uint16)
    o64 = np.empty((B, H, L, D), np.float64) if with_f64 else None
    for b in range(B):
        for h in range(H):
            r = sage_attention_head(q_bf16[b, h], k_bf16[b, h], v_bf16[b, h], scale, with_f64)
            if with_f64:
                out[b, h], o64[b, h] = r
            else:
                out[b, h] = r
    return (out, o64) if with_f64 else out
