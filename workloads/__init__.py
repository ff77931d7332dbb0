"""Seeded synthetic workloads shared by the CUDA path's tests/bench and the CPU oracle.

This package holds shapes and random numbers only: none of the method's
arithmetic (no scoring, selection or attention) lives here, so both sides can
draw identical inputs from it without sharing any computation.
"""

from .configs import CONFIGS, Workload, get_config
from .generate import bf16_round_bits, generate, host_sizes_for

__all__ = ["CONFIGS", "Workload", "get_config", "generate", "host_sizes_for", "bf16_round_bits"]
