"""The C-ABI libraries load, export every symbol their headers declare, and
reject bad arguments synchronously -- all without a GPU (no compute calls)."""
import ctypes
import os
import re

import pytest

from exact_io_aware_52_b200 import _binding as fb
from exact_io_aware_52_b200 import build as fbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared(header: str):
    text = open(os.path.join(ROOT, "include", header)).read()
    return re.findall(r"^FA_\w*EXPORT\s+[\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)


@pytest.fixture(scope="module", autouse=True)
def built():
    fbuild.build()


@pytest.mark.parametrize("header,lib", [("fa.h", fb.LIB_PATH), ("fa_selftest.h", fb.SELFTEST_LIB_PATH)])
def test_exports_every_declared_symbol(header, lib):
    names = declared(header)
    assert len(names) >= 4
    dll = ctypes.CDLL(lib)
    for n in names:
        assert hasattr(dll, n), f"{os.path.basename(lib)} does not export {n}"


def test_hidden_internals():
    dll = ctypes.CDLL(fb.LIB_PATH)
    assert not hasattr(dll, "validate")
    assert not hasattr(dll, "encode_map")


def test_status_strings_and_version():
    names = {0: "FA_OK", 1: "FA_ERR_INVALID_ARGUMENT", 2: "FA_ERR_MISALIGNED", 3: "FA_ERR_UNSUPPORTED",
             4: "FA_ERR_CUDA", 5: "FA_ERR_DEVICE_TIMEOUT", 6: "FA_ERR_WORKSPACE_LIMIT"}
    for code, name in names.items():
        assert fb.status_string(code) == name
    assert fb.status_string(99) == "FA_ERR_UNKNOWN"
    assert fb.version() == 300


def _params(**kw):
    base = dict(q=0x10000, k=0x20000, v=0x30000, o=0x40000, lse=0x50000, k_len=None, dev_status=None,
                B=1, H=2, N=128, d=64, causal=0, scale=0.125, o_dtype=0, flags=0, timeout_ms=0, H_kv=0,
                N_k=0, num_splits=0, workspace=None, workspace_bytes=0, in_dtype=0, descale_q=0.0, descale_k=0.0,
                descale_v=0.0)
    base.update(kw)
    return fb.FaParams(**base)


def _ex(**kw):
    p = _params(**kw)
    return fb.load().fa_fwd_ex(ctypes.byref(p), None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(k=None), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(v=None), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(o=None), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(lse=None), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(B=-1), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(H=-3), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(N=-128), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(scale=0.0), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(scale=-0.1), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(scale=float("nan")), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(scale=float("inf")), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(causal=2), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(o_dtype=7), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(flags=0x80), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(H_kv=-1), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(H=6, H_kv=4), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(H=6, H_kv=7), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(N_k=-1), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(num_splits=-2), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(num_splits=5000), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(N_k=1024, num_splits=4), fb.FA_ERR_INVALID_ARGUMENT),              # no workspace
    (dict(N_k=1024, num_splits=4, workspace=0x80000, workspace_bytes=64), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(N_k=1024, num_splits=4, workspace=0x80008, workspace_bytes=1 << 30), fb.FA_ERR_MISALIGNED),
    (dict(d=32), fb.FA_ERR_UNSUPPORTED),
    (dict(in_dtype=2), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(in_dtype=1, descale_q=-1.0), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(in_dtype=1, descale_v=float("nan")), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(descale_k=float("inf")), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(in_dtype=1, d=64), fb.FA_ERR_UNSUPPORTED),               # E4M3 inputs: d = 128 only
    (dict(in_dtype=1, d=256), fb.FA_ERR_UNSUPPORTED),
    (dict(d=512), fb.FA_ERR_UNSUPPORTED),
    (dict(d=192), fb.FA_ERR_UNSUPPORTED),
    (dict(d=96), fb.FA_ERR_UNSUPPORTED),
    (dict(q=0x10008), fb.FA_ERR_MISALIGNED),
    (dict(k=0x20004), fb.FA_ERR_MISALIGNED),
    (dict(v=0x30002), fb.FA_ERR_MISALIGNED),
    (dict(o=0x40001), fb.FA_ERR_MISALIGNED),
    (dict(lse=0x50002), fb.FA_ERR_MISALIGNED),
    (dict(k_len=0x60001), fb.FA_ERR_MISALIGNED),
    (dict(dev_status=0x70003), fb.FA_ERR_MISALIGNED),
    # empty problems are a no-op even with NULL buffers
    (dict(B=0, q=None, k=None, v=None, o=None, lse=None), fb.FA_OK),
    (dict(H=0), fb.FA_OK),
    (dict(N=0), fb.FA_OK),
])
def test_argument_errors_are_synchronous(kw, expect):
    # none of these reaches the device: the pointers are never dereferenced
    assert _ex(**kw) == expect


def test_workspace_bytes():
    lib = fb.load()
    p = _params(N_k=1000, num_splits=4)        # 8 key tiles -> 4 splits of 2 tiles
    assert lib.fa_fwd_workspace_bytes(ctypes.byref(p)) == 4 * (1 * 2 * 128) * (64 + 1) * 4
    p = _params(N_k=1000, num_splits=5)        # 5 requested -> 4 non-empty splits of 2 tiles
    assert lib.fa_fwd_workspace_bytes(ctypes.byref(p)) == 4 * (1 * 2 * 128) * (64 + 1) * 4
    p = _params(N_k=100, num_splits=8)         # one key tile: no split
    assert lib.fa_fwd_workspace_bytes(ctypes.byref(p)) == 0
    assert lib.fa_fwd_workspace_bytes(ctypes.byref(_params())) == 0
    assert lib.fa_fwd_workspace_bytes(None) == 0


def test_fa_fwd_validates_like_ex():
    lib = fb.load()
    f = ctypes.c_float
    assert lib.fa_fwd(None, 0x20000, 0x30000, 0x40000, 0x50000, 1, 1, 128, 64, 0, f(0.125), None) == \
        fb.FA_ERR_INVALID_ARGUMENT
    assert lib.fa_fwd(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 1, 1, 128, 80, 0, f(0.125), None) == \
        fb.FA_ERR_UNSUPPORTED
    assert lib.fa_fwd(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 1, 1, 0, 64, 1, f(0.125), None) == fb.FA_OK


def test_static_workspace_entry_validates():
    lib = fb.load()
    assert lib.fa_fwd_static_workspace(None, None) == fb.FA_ERR_INVALID_ARGUMENT
    # splits needing more than the fixed array: rejected before any CUDA call
    p = _params(H=8, N=1024, d=128, N_k=4096, num_splits=16)
    assert lib.fa_fwd_workspace_bytes(ctypes.byref(p)) > fb.FA_STATIC_WORKSPACE_BYTES
    assert lib.fa_fwd_static_workspace(ctypes.byref(p), None) == fb.FA_ERR_WORKSPACE_LIMIT
    # without splits it is fa_fwd_ex: the same synchronous argument errors
    assert lib.fa_fwd_static_workspace(ctypes.byref(_params(d=32)), None) == fb.FA_ERR_UNSUPPORTED
    assert lib.fa_fwd_static_workspace(ctypes.byref(_params(q=None)), None) == fb.FA_ERR_INVALID_ARGUMENT
    assert lib.fa_fwd_static_workspace(ctypes.byref(_params(N=0)), None) == fb.FA_OK
    # with splits, the argument checks still come first and make no CUDA call
    # (on a host without a GPU a CUDA call would turn these into FA_ERR_CUDA)
    assert lib.fa_fwd_static_workspace(ctypes.byref(_params(q=None, num_splits=4)), None) == \
        fb.FA_ERR_INVALID_ARGUMENT
    assert lib.fa_fwd_static_workspace(ctypes.byref(_params(num_splits=2000)), None) == fb.FA_ERR_INVALID_ARGUMENT
    assert lib.fa_fwd_static_workspace(ctypes.byref(_params(o=0x40008, num_splits=4)), None) == \
        fb.FA_ERR_MISALIGNED
    assert lib.fa_fwd_static_workspace(ctypes.byref(_params(d=32, num_splits=4)), None) == fb.FA_ERR_UNSUPPORTED


def test_host_entry_validates():
    lib = fb.load()
    assert lib.fa_fwd_host(None, None) == fb.FA_ERR_INVALID_ARGUMENT
    hp = fb.FaHostParams(q=None, k=0x1, v=0x1, k_len=None, o=0x1, lse=0x1, dev=_params())
    assert lib.fa_fwd_host(ctypes.byref(hp), None) == fb.FA_ERR_INVALID_ARGUMENT
    # host k_len without a device k_len buffer
    hp = fb.FaHostParams(q=0x1, k=0x1, v=0x1, k_len=0x1, o=0x1, lse=0x1, dev=_params())
    assert lib.fa_fwd_host(ctypes.byref(hp), None) == fb.FA_ERR_INVALID_ARGUMENT
    assert lib.fa_read_device_status(None, None) == fb.FA_ERR_INVALID_ARGUMENT


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(fb, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(fb, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        fb.load()


def _bwd_params(**kw):
    base = dict(q=0x10000, k=0x20000, v=0x30000, o=0x40000, dout=0x50000, lse=0x60000, dq=0x70000, dk=0x80000,
                dv=0x90000, k_len=None, dev_status=None, B=1, H=2, N=128, d=64, causal=0, scale=0.125, o_dtype=0,
                timeout_ms=0, H_kv=0, N_k=0, workspace=0xA0000, workspace_bytes=1 << 20)
    base.update(kw)
    return fb.FaBwdParams(**base)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(dout=None), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(dq=None), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(workspace=None), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(workspace_bytes=100), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(scale=0.0), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(causal=3), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(H_kv=3), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(N_k=-1), fb.FA_ERR_INVALID_ARGUMENT),
    (dict(d=256), fb.FA_ERR_UNSUPPORTED),
    (dict(dq=0x70008), fb.FA_ERR_MISALIGNED),
    (dict(workspace=0xA0004), fb.FA_ERR_MISALIGNED),
    (dict(B=0, q=None), fb.FA_OK),
])
def test_bwd_argument_errors_are_synchronous(kw, expect):
    assert fb.load().fa_bwd(ctypes.byref(_bwd_params(**kw)), None) == expect


def test_bwd_workspace_bytes():
    lib = fb.load()
    assert lib.fa_bwd_workspace_bytes(ctypes.byref(_bwd_params(B=2, H=3, N=100))) == 2 * 3 * 100 * 4
    assert lib.fa_bwd_workspace_bytes(None) == 0
