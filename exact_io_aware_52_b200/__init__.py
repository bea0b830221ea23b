"""B200-native exact attention forward (FlashAttention-style) behind a C ABI.

The hot path lives in ``csrc/`` (hand-written sm_100a CUDA, built into
``libfa_sm100.so``); this package is a thin ctypes binding over that library
plus the seeded workload generator.  Nothing here computes attention on the
CPU: when the library is missing, calls fail loudly.
"""
from .workloads import WORKLOADS, Workload, make_inputs, sample_rows  # noqa: F401

__all__ = ["WORKLOADS", "Workload", "make_inputs", "sample_rows"]
