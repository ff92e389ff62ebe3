"""Seeded synthetic inputs for the quantized linear (DiT layer shapes).

This module only draws random numbers: it holds none of the quantization or
matmul arithmetic, so both the CUDA path and the CPU oracle can take their
inputs from it.  Recipe (one ``numpy.random.default_rng(seed)`` per case, in
this draw order):

1. x: float64 standard normals of shape [M, K].  If ``outlier_frac`` > 0,
   ``round(outlier_frac * K)`` distinct channels are drawn without replacement
   and multiplied by ``outlier_scale`` (DiT activations carry a few large
   channels).  Then x is cast to float32 and rounded to bf16 (nearest-even).
2. W: float64 normals times ``w_std`` of shape [N, K], cast to float32.
3. bias (when requested): float64 normals times ``b_std`` of shape [N], float32.

Gated residual epilogue inputs (``gated_inputs``), from their own generator
``default_rng(seed + 1)``: the gate, float64 normals times 0.5 of shape [N]
with every 7th channel set to 0 (closed), cast to float32; then the residual
rows, float64 normals of shape [rows, N] cast to float32 and rounded to bf16.

bf16 arrays are returned as numpy uint16 bit patterns.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even) and return the bit patterns.

    torch's CPU cast does the rounding; it is only used to make the input tensor.
    """
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@dataclass
class LinearCase:
    name: str
    M: int
    K: int
    N: int
    x_std: float = 1.0
    outlier_frac: float = 0.0
    outlier_scale: float = 20.0
    w_std: float = 0.02
    bias: bool = True
    b_std: float = 0.1
    seed: int = 0
    extra: dict = field(default_factory=dict)

    def draw(self):
        """Return (x bf16 bits [M,K], W float32 [N,K], bias float32 [N] or None, outlier channels)."""
        rng = np.random.default_rng(self.seed)
        x = rng.standard_normal((self.M, self.K)) * self.x_std
        chans = np.empty(0, np.int64)
        if self.outlier_frac > 0:
            n_out = int(round(self.outlier_frac * self.K))
            chans = np.sort(rng.choice(self.K, size=n_out, replace=False))
            x[:, chans] *= self.outlier_scale
        x_bf16 = f32_to_bf16_bits(x.astype(np.float32))
        del x
        W = (rng.standard_normal((self.N, self.K)) * self.w_std).astype(np.float32)
        b = None
        if self.bias:
            b = (rng.standard_normal(self.N) * self.b_std).astype(np.float32)
        return x_bf16, W, b, chans


def gated_inputs(case: LinearCase, rows: int | None = None):
    """(gate float32 [N], residual bf16 bits [rows, N]) for the gated residual
    epilogue of `case` (first `rows` rows of the residual; all M by default)."""
    rng = np.random.default_rng(case.seed + 1)
    gate = rng.standard_normal(case.N) * 0.5
    gate[::7] = 0.0
    rows = case.M if rows is None else rows
    res = np.empty((rows, case.N), np.uint16)
    step = max(1, (1 << 24) // max(case.N, 1))  # bounded host memory per block
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        res[r0:r1] = f32_to_bf16_bits(rng.standard_normal((r1 - r0, case.N)).astype(np.float32))
    return gate.astype(np.float32), res


# The five workloads of the quantized linear, at DiT layer shapes.
TINY = LinearCase("tiny_w8a8_64x256x128", M=64, K=256, N=128)
DIT_ATTN = LinearCase("dit_attn_proj_w8a8_4096x3072x3072", M=4096, K=3072, N=3072,
                      outlier_frac=0.01)
SWEEP = [
    LinearCase("sweep_w8a8_2048x4096x4096", M=2048, K=4096, N=4096),
    LinearCase("sweep_w8a8_2048x4096x12288", M=2048, K=4096, N=12288),
    LinearCase("sweep_w8a8_2048x12288x4096", M=2048, K=12288, N=4096),
    LinearCase("sweep_w8a8_2048x5120x48_thin", M=2048, K=5120, N=48),
]
DIT_MLP = LinearCase("dit_mlp_w8a8_16384x3072x12288", M=16384, K=3072, N=12288,
                     outlier_frac=0.01)
W4A8 = [LinearCase(f"w4a8_g64_{m}x4096x4096", M=m, K=4096, N=4096, bias=False)
        for m in (1, 8, 16, 4096)]

# The quick-start matmul of the qlip-mlx README ("Quick start": 14040 tokens x
# 5120 @ 5120 x 5120, bf16 vs W8A8 vs W4A8 on bare tensors, no bias).
QUICKSTART = [LinearCase("quickstart_w8a8_14040x5120x5120", M=14040, K=5120, N=5120, bias=False),
              LinearCase("quickstart_w4a8_14040x5120x5120", M=14040, K=5120, N=5120, bias=False)]

@dataclass
class AttentionCase:
    """q, k, v bf16 [B, H, L, 128], float64 standard normals (q times q_std)
    from default_rng(seed) in the order q, k, v, rounded to bf16."""
    name: str
    B: int
    H: int
    L: int
    D: int = 128
    q_std: float = 1.0
    seed: int = 0

    def draw(self, heads=None):
        """(q, k, v) bf16 bits; `heads` limits the draw to the first heads."""
        rng = np.random.default_rng(self.seed)
        H = self.H if heads is None else heads
        shape = (self.B, H, self.L, self.D)
        out = []
        for std in (self.q_std, 1.0, 1.0):
            t = np.empty(shape, np.uint16)
            for h in range(H):  # bounded host memory per draw
                t[:, h] = f32_to_bf16_bits((rng.standard_normal((self.B, self.L, self.D)) * std)
                                           .astype(np.float32))
            out.append(t)
        return tuple(out)


# The README's quick-start attention (40 heads x 14040 tokens, head dim 128).
SAGE_QUICKSTART = AttentionCase("sage_attn_40x14040x128", B=1, H=40, L=14040)

ALL_W8A8 = [TINY, DIT_ATTN, *SWEEP, DIT_MLP]
