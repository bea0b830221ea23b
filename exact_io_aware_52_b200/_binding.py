"""ctypes binding over the C ABI of include/fa.h (libfa_sm100.so).

Argument marshalling only: tensors are passed as raw device pointers and the
current CUDA stream; every step of the computation runs in the CUDA library.
torch supplies device memory and streams.  If the library is missing, every
call raises -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa_sm100.so")
SELFTEST_LIB_PATH = os.path.join(HERE, "libfa_selftest.so")

FA_OK = 0
FA_ERR_INVALID_ARGUMENT = 1
FA_ERR_MISALIGNED = 2
FA_ERR_UNSUPPORTED = 3
FA_ERR_CUDA = 4
FA_ERR_DEVICE_TIMEOUT = 5
FA_ERR_WORKSPACE_LIMIT = 6
FA_ERR_SCHED_BUSY = 7
FA_STATIC_WORKSPACE_BYTES = 64 * 1024 * 1024   # include/fa.h
FA_O_F32 = 0
FA_O_BF16 = 1
FA_IN_BF16 = 0
FA_IN_E4M3 = 1
FA_FLAG_EAGER_RESCALE = 1

_lock = threading.Lock()
_lib = None
_selftest = None


class FaParams(ctypes.Structure):
    """Mirror of fa_fwd_params."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("k_len", ctypes.c_void_p),
        ("dev_status", ctypes.c_void_p),
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
        ("causal", ctypes.c_int), ("scale", ctypes.c_float), ("o_dtype", ctypes.c_int),
        ("flags", ctypes.c_int), ("timeout_ms", ctypes.c_uint32), ("H_kv", ctypes.c_int),
        ("N_k", ctypes.c_int), ("num_splits", ctypes.c_int), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t), ("in_dtype", ctypes.c_int), ("descale_q", ctypes.c_float),
        ("descale_k", ctypes.c_float), ("descale_v", ctypes.c_float), ("test_drop_load", ctypes.c_int),
    ]


class FaHostParams(ctypes.Structure):
    """Mirror of fa_fwd_host_params."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("k_len", ctypes.c_void_p), ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("dev", FaParams),
    ]


class FaBwdParams(ctypes.Structure):
    """Mirror of fa_bwd_params (include/fa.h)."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("o", ctypes.c_void_p),
        ("dout", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p),
        ("dv", ctypes.c_void_p), ("k_len", ctypes.c_void_p), ("dev_status", ctypes.c_void_p),
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
        ("causal", ctypes.c_int), ("scale", ctypes.c_float), ("o_dtype", ctypes.c_int),
        ("timeout_ms", ctypes.c_uint32), ("H_kv", ctypes.c_int), ("N_k", ctypes.c_int),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
    ]


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where} failed: {status_string(status)} ({status})")


def load():
    """Load libfa_sm100.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                                   "(run `python -m exact_io_aware_52_b200.build`)")
            lib = ctypes.CDLL(LIB_PATH)
            vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
            lib.fa_fwd.restype = i
            lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
            lib.fa_fwd_ex.restype = i
            lib.fa_fwd_ex.argtypes = [ctypes.POINTER(FaParams), vp]
            lib.fa_fwd_host.restype = i
            lib.fa_fwd_host.argtypes = [ctypes.POINTER(FaHostParams), vp]
            lib.fa_read_device_status.restype = i
            lib.fa_read_device_status.argtypes = [vp, vp]
            lib.fa_status_string.restype = ctypes.c_char_p
            lib.fa_status_string.argtypes = [i]
            lib.fa_version.restype = i
            lib.fa_version.argtypes = []
            lib.fa_fwd_workspace_bytes.restype = ctypes.c_size_t
            lib.fa_fwd_workspace_bytes.argtypes = [ctypes.POINTER(FaParams)]
            lib.fa_fwd_suggest_splits.restype = i
            lib.fa_fwd_suggest_splits.argtypes = [ctypes.POINTER(FaParams)]
            lib.fa_bwd.restype = i
            lib.fa_bwd.argtypes = [ctypes.POINTER(FaBwdParams), ctypes.c_void_p]
            lib.fa_bwd_workspace_bytes.restype = ctypes.c_size_t
            lib.fa_bwd_workspace_bytes.argtypes = [ctypes.POINTER(FaBwdParams)]
            lib.fa_fwd_static_workspace.restype = i
            lib.fa_fwd_static_workspace.argtypes = [ctypes.POINTER(FaParams), ctypes.c_void_p]
            lib.fa_testhook_sched_next_slot.restype = i
            lib.fa_testhook_sched_next_slot.argtypes = []
            lib.fa_testhook_sched_slot.restype = i
            lib.fa_testhook_sched_slot.argtypes = [i, vp, vp]
            _lib = lib
    return _lib


def load_selftest():
    """Load libfa_selftest.so (raises if it has not been built)."""
    global _selftest
    with _lock:
        if _selftest is None:
            if not os.path.exists(SELFTEST_LIB_PATH):
                raise RuntimeError(f"self-test library not built: {SELFTEST_LIB_PATH} is missing")
            lib = ctypes.CDLL(SELFTEST_LIB_PATH)
            vp, i = ctypes.c_void_p, ctypes.c_int
            lib.fa_selftest_tma_sw128.restype = i
            lib.fa_selftest_tma_sw128.argtypes = [vp, vp, vp, vp]
            lib.fa_selftest_mma_ss.restype = i
            lib.fa_selftest_mma_ss.argtypes = [vp, vp, vp, i, vp, vp]
            lib.fa_selftest_mma_ts.restype = i
            lib.fa_selftest_mma_ts.argtypes = [vp, vp, vp, i, vp, vp]
            lib.fa_selftest_mma_e4m3_ss.restype = i
            lib.fa_selftest_mma_e4m3_ss.argtypes = [vp, vp, vp, vp, vp]
            lib.fa_selftest_mma_e4m3_ts.restype = i
            lib.fa_selftest_mma_e4m3_ts.argtypes = [vp, vp, vp, vp, vp]
            lib.fa_selftest_exp2_poly.restype = i
            lib.fa_selftest_exp2_poly.argtypes = [vp, vp, i, vp]
            lib.fa_selftest_mufu_rate.restype = i
            lib.fa_selftest_mufu_rate.argtypes = [i, i, i, ctypes.POINTER(ctypes.c_double), vp]
            lib.fa_selftest_wait_timeout.restype = i
            lib.fa_selftest_wait_timeout.argtypes = [vp, ctypes.c_uint32, vp]
            _selftest = lib
    return _selftest


def status_string(status: int) -> str:
    return load().fa_status_string(int(status)).decode()


def version() -> int:
    return load().fa_version()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(st: int, where: str):
    if st != FA_OK:
        raise FaError(st, where)


def fa_fwd(q, k, v, o, lse, causal: bool, scale: float, stream=None):
    """fa_fwd: q, k, v bf16 [B,H,N,d] CUDA tensors; o fp32 [B,H,N,d]; lse fp32 [B,H,N]."""
    B, H, N, d = q.shape
    st = load().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, int(bool(causal)),
                       ctypes.c_float(scale), _stream(stream))
    _check(st, "fa_fwd")


def make_params(q, k, v, o, lse, causal, scale, k_len=None, dev_status=None, flags=0, timeout_ms=0,
                shape=None, num_splits=0, workspace=None, descale=(0.0, 0.0, 0.0), test_drop_load=0) -> FaParams:
    """Fill a fa_fwd_params from tensors (any of them may be None for argument tests).

    k, v may be [B, H_kv, N_k, d] with H_kv dividing H and any N_k; workspace is a
    CUDA tensor of at least workspace_bytes(...) bytes when num_splits > 1.
    q, k, v of dtype torch.float8_e4m3fn select E4M3 inputs, whose values are
    scaled by descale = (descale_q, descale_k, descale_v) (0 means 1)."""
    import torch
    if shape is None:
        shape = tuple(q.shape)
    B, H, N, d = shape
    o_dtype = FA_O_BF16 if (o is not None and o.dtype == torch.bfloat16) else FA_O_F32
    kv4 = k is not None and hasattr(k, "shape") and k.dim() == 4
    H_kv = int(k.shape[1]) if kv4 else 0
    N_k = int(k.shape[2]) if kv4 else 0
    if kv4 and N_k == 0 and B * H * N > 0:
        # N_k = 0 means "N keys" in the C ABI; an empty key tensor is key padding (k_len = 0)
        raise ValueError("k and v have no keys: pass at least one key row and k_len = 0")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return FaParams(q=_ptr(q), k=_ptr(k), v=_ptr(v), o=_ptr(o), lse=_ptr(lse), k_len=_ptr(k_len),
                    dev_status=_ptr(dev_status), B=B, H=H, N=N, d=d, causal=int(bool(causal)),
                    scale=float(scale), o_dtype=o_dtype, flags=int(flags), timeout_ms=int(timeout_ms),
                    H_kv=H_kv, N_k=N_k, num_splits=int(num_splits), workspace=_ptr(workspace),
                    workspace_bytes=ws_bytes,
                    in_dtype=FA_IN_E4M3 if getattr(q, "dtype", None) == torch.float8_e4m3fn else FA_IN_BF16,
                    descale_q=float(descale[0]), descale_k=float(descale[1]), descale_v=float(descale[2]),
                    test_drop_load=int(test_drop_load))


def workspace_bytes(q, k, num_splits: int) -> int:
    """Scratch bytes a num_splits > 1 call needs (fa_fwd_workspace_bytes)."""
    p = make_params(q, k, None, None, None, False, 1.0, num_splits=num_splits)
    return int(load().fa_fwd_workspace_bytes(ctypes.byref(p)))


def suggest_splits(q, k) -> int:
    """The library's key-split count for this shape on the current device."""
    p = make_params(q, k, None, None, None, False, 1.0)
    return int(load().fa_fwd_suggest_splits(ctypes.byref(p)))


def fa_fwd_ex(q, k, v, o, lse, causal: bool, scale: float, k_len=None, dev_status=None, flags: int = 0,
              timeout_ms: int = 0, stream=None, num_splits: int = 0, workspace=None, descale=(0.0, 0.0, 0.0),
              test_drop_load: int = 0):
    """fa_fwd_ex: as fa_fwd, plus k_len (int32 [B] CUDA tensor), o may be bf16,
    an optional int32 status word, FA_FLAG_* flags and the wait time limit.
    k and v may be [B, H_kv, N_k, d] (grouped heads, more keys than queries);
    num_splits > 1 splits each row's keys, with `workspace` as scratch."""
    p = make_params(q, k, v, o, lse, causal, scale, k_len, dev_status, flags, timeout_ms,
                    num_splits=num_splits, workspace=workspace, descale=descale, test_drop_load=test_drop_load)
    _check(load().fa_fwd_ex(ctypes.byref(p), _stream(stream)), "fa_fwd_ex")


def fa_fwd_static_workspace(q, k, v, o, lse, causal: bool, scale: float, k_len=None, dev_status=None,
                            flags: int = 0, timeout_ms: int = 0, stream=None, num_splits: int = 0,
                            descale=(0.0, 0.0, 0.0)):
    """fa_fwd_static_workspace: fa_fwd_ex with the split scratch in the library's
    fixed device array (FA_STATIC_WORKSPACE_BYTES per device, shared by all calls
    on the device: do not overlap calls).  Allocates nothing."""
    p = make_params(q, k, v, o, lse, causal, scale, k_len, dev_status, flags, timeout_ms, num_splits=num_splits,
                    descale=descale)
    _check(load().fa_fwd_static_workspace(ctypes.byref(p), _stream(stream)), "fa_fwd_static_workspace")


def fa_fwd_host(q_h, k_h, v_h, o_h, lse_h, q_d, k_d, v_d, o_d, lse_d, causal: bool, scale: float,
                k_len_h=None, k_len_d=None, dev_status=None, flags: int = 0, stream=None, num_splits: int = 0,
                workspace=None, descale=(0.0, 0.0, 0.0)):
    """fa_fwd_host: host (pinned) tensors in and out, device tensors as staging."""
    dev = make_params(q_d, k_d, v_d, o_d, lse_d, causal, scale, k_len_d, dev_status, flags,
                      num_splits=num_splits, workspace=workspace, descale=descale)
    hp = FaHostParams(q=_ptr(q_h), k=_ptr(k_h), v=_ptr(v_h), k_len=_ptr(k_len_h), o=_ptr(o_h), lse=_ptr(lse_h),
                      dev=dev)
    _check(load().fa_fwd_host(ctypes.byref(hp), _stream(stream)), "fa_fwd_host")


def read_device_status(dev_status, stream=None) -> int:
    return load().fa_read_device_status(_ptr(dev_status), _stream(stream))


def attention(q, k, v, causal: bool, scale: float, k_len=None, out_dtype=None, flags: int = 0, stream=None,
              num_splits: int = 0, descale=(0.0, 0.0, 0.0)):
    """Allocate O, lse (and any split workspace) with torch on q's device and run fa_fwd_ex.

    num_splits: 0 = none, -1 = the library's suggestion, S > 1 = S key splits.
    Returns (O [B,H,N,d] in out_dtype (fp32 default), lse [B,H,N] fp32).
    """
    import torch
    B, H, N, d = q.shape
    o = torch.empty((B, H, N, d), dtype=out_dtype or torch.float32, device=q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if num_splits < 0:
        num_splits = suggest_splits(q, k)
    ws = None
    if num_splits > 1:
        ws = torch.empty(max(workspace_bytes(q, k, num_splits), 16), dtype=torch.uint8, device=q.device)
    fa_fwd_ex(q, k, v, o, lse, causal, scale, k_len=k_len, flags=flags, stream=stream, num_splits=num_splits,
              workspace=ws, descale=descale)
    return o, lse


def make_bwd_params(q, k, v, o, lse, dout, dq, dk, dv, causal, scale, k_len=None, dev_status=None, timeout_ms=0,
                    workspace=None, shape=None) -> FaBwdParams:
    """Fill a fa_bwd_params from tensors (q, dout, o, dq [B, H, N, d]; k, v, dk, dv
    [B, H_kv, N_k, d]; lse [B, H, N])."""
    import torch
    if shape is None:
        shape = tuple(q.shape)
    B, H, N, d = shape
    kv4 = k is not None and hasattr(k, "shape") and k.dim() == 4
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return FaBwdParams(q=_ptr(q), k=_ptr(k), v=_ptr(v), o=_ptr(o), dout=_ptr(dout), lse=_ptr(lse), dq=_ptr(dq),
                       dk=_ptr(dk), dv=_ptr(dv), k_len=_ptr(k_len), dev_status=_ptr(dev_status), B=B, H=H, N=N,
                       d=d, causal=int(bool(causal)), scale=float(scale),
                       o_dtype=FA_O_BF16 if (o is not None and o.dtype == torch.bfloat16) else FA_O_F32,
                       timeout_ms=int(timeout_ms), H_kv=int(k.shape[1]) if kv4 else 0,
                       N_k=int(k.shape[2]) if kv4 else 0, workspace=_ptr(workspace), workspace_bytes=ws_bytes)


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, causal: bool, scale: float, workspace, k_len=None, dev_status=None,
           timeout_ms: int = 0, stream=None):
    """fa_bwd: gradients dq, dk, dv (fp32 CUDA tensors, overwritten) of the forward
    (o, lse) for dout; workspace: CUDA tensor of >= fa_bwd_workspace_bytes bytes."""
    p = make_bwd_params(q, k, v, o, lse, dout, dq, dk, dv, causal, scale, k_len, dev_status, timeout_ms, workspace)
    _check(load().fa_bwd(ctypes.byref(p), _stream(stream)), "fa_bwd")


def bwd_workspace_bytes(q) -> int:
    B, H, N, _ = q.shape
    return 4 * B * H * N


def attention_bwd(q, k, v, o, lse, dout, causal: bool, scale: float, k_len=None, stream=None):
    """Allocate dq, dk, dv (fp32) and the workspace with torch on q's device and run fa_bwd."""
    import torch
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    ws = torch.empty(max(bwd_workspace_bytes(q), 16), dtype=torch.uint8, device=q.device)
    fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, causal, scale, ws, k_len=k_len, stream=stream)
    return dq, dk, dv
