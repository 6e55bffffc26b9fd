"""Group-wise fully quantized int8 Winograd convolution F(m,3) for NVIDIA B200 (sm_100a).

The product is the C-ABI CUDA library (include/wino.h, built in-tree as
libwino_b200.so); `wino` is its thin ctypes binding and `synth` holds the
seeded synthetic layers used by the tests and the benchmark.
"""
from . import synth  # noqa: F401

__all__ = ["synth", "wino", "build"]
