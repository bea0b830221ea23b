"""Build the sm_100a CUDA library ``libfa_sm100.so`` in-tree with nvcc.

    python -m exact_io_aware_52_b200.build [--verbose]

Cross-compiles without a GPU.  The library exports the C ABI of include/fa.h.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libfa_sm100.so")
SELFTEST_LIB = os.path.join(HERE, "libfa_selftest.so")
# library -> its translation units
TARGETS = {
    LIB: [os.path.join(CSRC, "fa_api.cu"), os.path.join(CSRC, "fa_static_workspace.cu")],
    SELFTEST_LIB: [os.path.join(CSRC, "selftest.cu")],
}
HEADERS = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + \
    [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _build_one(lib: str, srcs: list, force: bool, verbose: bool) -> str:
    if not force and os.path.exists(lib):
        t = os.path.getmtime(lib)
        if all(os.path.getmtime(f) <= t for f in [*srcs, *HEADERS]):
            return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-shared", "-I", INCLUDE, "-I", CSRC, *srcs, "-o", tmp, "-lcudart"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> list:
    """Compile every library that is older than its sources; returns their paths."""
    return [_build_one(lib, srcs, force, verbose) for lib, srcs in TARGETS.items()]


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
