"""Shared test helpers: bf16 distance, tensor <-> numpy, sampled rows."""
import numpy as np


def ordinal(bits):
    """bf16 bit patterns -> integers monotone in the value (+0 and -0 both 0)."""
    b = np.asarray(bits, np.uint16).astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def bf16_ulp_distance(a_bits, b_bits):
    return np.abs(ordinal(a_bits) - ordinal(b_bits))


def t2bits(t):
    """torch bf16/fp16 tensor (any device) -> numpy uint16 bit patterns."""
    import torch

    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bits2t(bits, dtype, device):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(dtype).to(device)


def sample_rows(M, tile=128, extra=8, seed=0):
    """Rows that cover the first/last row of several M tiles, the ragged tail and
    some random rows."""
    rng = np.random.default_rng(seed)
    rows = {0, M - 1}
    for t in range(0, M, tile):
        rows.update({t, min(t + tile - 1, M - 1)})
        if len(rows) > 24:
            break
    rows.update(int(r) for r in rng.integers(0, M, size=extra))
    return np.array(sorted(rows), np.int64)
