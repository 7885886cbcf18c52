"""Seeded synthetic inputs shared by the tests, the benchmark and the checker.

Holds random-number generation and workload shapes only, never the arithmetic
of the method under test.
"""
from .workloads import *  # noqa: F401,F403
from .philox import philox4x32, approx_normal_from_words, f32_to_bf16_bits, bf16_bits_to_f32  # noqa: F401
