"""fp64 CPU oracle for the exact attention forward pass.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA product path
never imports this package, and this package imports nothing from it.

Three pieces, all written from the page "FlashAttention (ES)":

* ``attention_f64`` -- the plain definition of attention (section "El problema
  de la atencion estandar", the Attention equation, with the masking step of
  section "Fusion de operaciones en un unico kernel de CUDA"), computed in C
  with OpenMP over rows in ``attn_oracle.c``: full score row, mask,
  max-subtracted softmax, weighted sum of V rows.
* ``attention_bwd_f64`` -- the gradients dQ, dK, dV of that definition for a
  given dO (the chain rule through the row softmax; the pages give no
  backward algorithm), in C with OpenMP over key/value heads in
  ``attn_bwd_oracle.c``.
* ``online.attention_online`` -- the tiled online-softmax recurrence of
  section "Calculo de Softmax en linea" in pure Python, used only on tiny
  inputs to pin the recurrence against the two-pass definition.

Pinned by ``tests/test_oracle.py`` against closed forms, invariants, a
library routine (torch's fp64 scaled-dot-product attention) and brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_BWD_SRC = os.path.join(_HERE, "attn_bwd_oracle.c")
_BWD_LIB = os.path.join(_HERE, "liboracle_bwd.so")
_lock = threading.Lock()
_lib = None
_bwd_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the C oracle (``attn_oracle.c`` by default) into a shared library.

    No fast-math: the oracle keeps IEEE double semantics.
    """
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
             "-fno-fast-math", src, "-o", tmp, "-lm"])
        os.replace(tmp, out)
    return out


def load_library(path: str):
    """ctypes handle on a built oracle library with its signature declared."""
    lib = ctypes.CDLL(path)
    f = lib.attn_oracle_f64
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_void_p,
                  ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(build())
    return _lib


def build_bwd(force: bool = False, src: str = _BWD_SRC, out: str = _BWD_LIB) -> str:
    """Compile the backward oracle (``attn_bwd_oracle.c`` by default)."""
    return build(force=force, src=src, out=out)


def load_bwd_library(path: str):
    """ctypes handle on a built backward-oracle library with its signature declared."""
    lib = ctypes.CDLL(path)
    f = lib.attn_bwd_oracle_f64
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 7 + [ctypes.c_float] + [ctypes.c_void_p] * 3 + \
        [ctypes.c_int]
    return lib


def _load_bwd():
    global _bwd_lib
    with _lock:
        if _bwd_lib is None:
            _bwd_lib = load_bwd_library(build_bwd())
    return _bwd_lib


def _as_bf16_bits(x) -> np.ndarray:
    """Accept a torch bf16 tensor (CPU) or a numpy uint16 array of bf16 bits."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy inputs must be uint16 bf16 bit patterns")
        return np.ascontiguousarray(x)
    import torch  # only for the bit view of a bf16 tensor
    if x.dtype != torch.bfloat16:
        raise TypeError("torch inputs must be bfloat16")
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def attention_f64(q, k, v, causal: bool, scale: float, k_len=None, rows=None,
                  nthreads: int | None = None, lib=None):
    """Exact attention in fp64 from bf16 inputs.

    q: [B, H, N, d] and k, v: [B, H_kv, Nk, d] bf16 (torch CPU tensors or uint16
    bit arrays); H_kv divides H and query head h uses key/value head h // (H // H_kv);
    with Nk keys query i sits at key position i + Nk - N (causal: key j <= i + Nk - N).
    causal: key j is masked for query i when j > i.
    scale: the float32 multiplier of q.k (the definition's 1/sqrt(d_k)).
    k_len: None or int sequence of length B; key j of batch b masked iff j >= k_len[b].
    rows: None (all rows) or int64 flat row ids (b*H + h)*N + i.
    lib: a library from ``load_library`` (default: the built ``attn_oracle.c``).
    Returns (O [n_rows, d] float64, lse [n_rows] float64); n_rows = B*H*N when
    rows is None (row r = (b*H + h)*N + i).
    """
    qb, kb, vb = _as_bf16_bits(q), _as_bf16_bits(k), _as_bf16_bits(v)
    if qb.ndim != 4 or kb.ndim != 4 or kb.shape != vb.shape:
        raise ValueError("q must be [B, H, N, d] and k, v [B, H_kv, N, d]")
    B, H, N, d = qb.shape
    H_kv, Nk = kb.shape[1], kb.shape[2]
    if (kb.shape[0], kb.shape[3]) != (B, d) or H_kv == 0 or H % H_kv:
        raise ValueError("k, v must be [B, H_kv, Nk, d] with H_kv dividing H")
    kl = None
    if k_len is not None:
        kl = np.ascontiguousarray(np.asarray(k_len, dtype=np.int32).reshape(-1))
        if kl.shape[0] != B:
            raise ValueError("k_len must have B entries")
    if rows is None:
        n_rows = B * H * N
        rr = None
    else:
        rr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
        n_rows = rr.shape[0]
    o = np.zeros((n_rows, d), dtype=np.float64)
    lse = np.zeros((n_rows,), dtype=np.float64)
    nt = nthreads if nthreads is not None else (os.cpu_count() or 1)
    lib = _load() if lib is None else lib
    rc = lib.attn_oracle_f64(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data,
        None if kl is None else kl.ctypes.data, B, H, H_kv, N, Nk, d, int(bool(causal)),
        ctypes.c_float(scale), None if rr is None else rr.ctypes.data,
        n_rows, o.ctypes.data, lse.ctypes.data, int(nt))
    if rc != 0:
        raise RuntimeError(f"attn_oracle_f64 failed with code {rc}")
    return o, lse


def attention_bwd_f64(q, k, v, dout, causal: bool, scale: float, k_len=None, nthreads: int | None = None,
                      lib=None):
    """Gradients of exact attention in fp64 from bf16 inputs.

    q, dout: [B, H, N, d]; k, v: [B, H_kv, Nk, d] (bf16 torch CPU tensors or
    uint16 bit arrays), with the masks and head grouping of ``attention_f64``;
    dout is the gradient of the loss with respect to O.
    Returns (dq [B, H, N, d], dk [B, H_kv, Nk, d], dv [B, H_kv, Nk, d]) float64.
    """
    qb, kb, vb, db = _as_bf16_bits(q), _as_bf16_bits(k), _as_bf16_bits(v), _as_bf16_bits(dout)
    if qb.ndim != 4 or kb.shape != vb.shape or db.shape != qb.shape:
        raise ValueError("q, dout must be [B, H, N, d] and k, v [B, H_kv, Nk, d]")
    B, H, N, d = qb.shape
    H_kv, Nk = kb.shape[1], kb.shape[2]
    if (kb.shape[0], kb.shape[3]) != (B, d) or H_kv == 0 or H % H_kv:
        raise ValueError("k, v must be [B, H_kv, Nk, d] with H_kv dividing H")
    kl = None
    if k_len is not None:
        kl = np.ascontiguousarray(np.asarray(k_len, dtype=np.int32).reshape(-1))
        if kl.shape[0] != B:
            raise ValueError("k_len must have B entries")
    dq = np.zeros((B, H, N, d), dtype=np.float64)
    dk = np.zeros((B, H_kv, Nk, d), dtype=np.float64)
    dv = np.zeros((B, H_kv, Nk, d), dtype=np.float64)
    nt = nthreads if nthreads is not None else (os.cpu_count() or 1)
    lib = _load_bwd() if lib is None else lib
    rc = lib.attn_bwd_oracle_f64(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, db.ctypes.data,
        None if kl is None else kl.ctypes.data, B, H, H_kv, N, Nk, d, int(bool(causal)),
        ctypes.c_float(scale), dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, int(nt))
    if rc != 0:
        raise RuntimeError(f"attn_bwd_oracle_f64 failed with code {rc}")
    return dq, dk, dv
