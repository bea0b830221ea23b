"""B200-native exact attention forward (FlashAttention-style) behind a C ABI.

The hot path lives in ``csrc/`` (hand-written sm_100a CUDA built into
``libfa_sm100.so``, C ABI in ``include/fa.h``); this package is a thin ctypes
binding over that library plus the seeded workload generator.  Nothing here
computes attention on the CPU: when the library is missing, calls fail loudly.
"""
from ._binding import (  # noqa: F401
    FA_ERR_CUDA, FA_ERR_DEVICE_TIMEOUT, FA_ERR_INVALID_ARGUMENT, FA_ERR_MISALIGNED, FA_ERR_UNSUPPORTED,
    FA_ERR_WORKSPACE_LIMIT, FA_FLAG_EAGER_RESCALE, FA_IN_BF16, FA_IN_E4M3, FA_O_BF16, FA_O_F32, FA_OK, FA_STATIC_WORKSPACE_BYTES, FaError,
    attention, attention_bwd, fa_bwd, fa_fwd, fa_fwd_ex, fa_fwd_host, fa_fwd_static_workspace, read_device_status, status_string,
    suggest_splits, version, workspace_bytes,
)
from .workloads import WORKLOADS, Workload, make_inputs, sample_rows  # noqa: F401
