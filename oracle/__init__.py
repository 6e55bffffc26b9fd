"""CPU oracle for group-wise fully quantized int8 Winograd convolution.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline leg, never by the library.
"""
from .oracle import *  # noqa: F401,F403
