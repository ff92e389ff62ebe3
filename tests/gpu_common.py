"""Fixtures for the GPU parity tests (marked gpu; they need a B200)."""
import numpy as np
import pytest
import torch

from tests.helpers import bits2t, t2bits


@pytest.fixture(scope="session")
def qk():
    from w4a8_quantized_gemm_token_b200 import build

    build.build()
    from w4a8_quantized_gemm_token_b200 import binding

    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    assert binding.qk_is_available(torch.cuda.current_device()), "the library needs sm_100 (B200)"
    return binding


def to_dev_bf16(xb):
    return bits2t(xb, torch.bfloat16, "cuda")


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


__all__ = ["qk", "to_dev_bf16", "to_dev", "host", "t2bits", "bits2t"]
