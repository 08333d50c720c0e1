"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This package holds random-number generation and input recipes only: it does
none of the sparse-attention arithmetic (no scoring, selection, softmax or FP8
scaling rule of the method).  Both the CPU oracle and the CUDA path are fed
from here, so neither has to import the other.
"""
from .generators import (  # noqa: F401
    splitmix64_np, normal_np, normal_torch, uniform_np,
    bf16_bits_np, bf16_bits_torch, bf16_bits_to_f32_np,
    sub_seed, ar1_keys_np, e4m3_codes_torch, e4m3_codes_np, normal_bf16_torch,
)
from .workloads import *  # noqa: F401,F403
