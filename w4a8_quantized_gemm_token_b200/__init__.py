"""B200-native W8A8 / W4A8 quantized linear.

The compute lives in ``libqk.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/qk.h``).  ``binding`` is a thin ctypes layer over it with
the same function names.  ``synthetic`` draws the seeded DiT-shaped inputs.

Importing the package loads nothing; ``from w4a8_quantized_gemm_token_b200 import
binding`` loads the library and raises if it has not been built.
"""

__all__ = ["binding", "synthetic"]
