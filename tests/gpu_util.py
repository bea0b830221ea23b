"""Helpers shared by the GPU parity tests: run the CUDA path through the C
ABI and compare with the fp64 oracle at the parity tolerances."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from exact_io_aware_52_b200 import _binding as fb
from exact_io_aware_52_b200 import workloads

# parity tolerances for bf16 inputs with fp32 accumulation
TOL_MAX = 1e-2    # max |O_gpu - O_ref|
TOL_MEAN = 1e-3   # mean |O_gpu - O_ref|
TOL_LSE = 1e-4    # max |lse_gpu - lse_ref| / max(|lse_ref|, 1)


# Guard regions: every output buffer a GPU test hands to the library sits
# between two runs of GUARD_BYTES bytes of a fixed pattern, checked bit for bit
# after the call, so a store past either end of a buffer (a wrong row index, a
# ragged tail, a split layout off by one) fails the test instead of silently
# corrupting a neighbour.
GUARD_BYTES = 4096
GUARD_BYTE = 0xA5


class Guarded:
    """A device tensor of `shape` and `dtype` with guard bytes on both sides."""

    def __init__(self, shape, dtype, dev, fill=None):
        esize = torch.empty((), dtype=dtype).element_size()
        self.nbytes = int(np.prod(shape)) * esize
        self.buf = torch.full((2 * GUARD_BYTES + self.nbytes,), GUARD_BYTE, dtype=torch.uint8, device=dev)
        self.t = self.buf[GUARD_BYTES:GUARD_BYTES + self.nbytes].view(dtype).view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self, name="buffer"):
        head = self.buf[:GUARD_BYTES]
        tail = self.buf[GUARD_BYTES + self.nbytes:]
        bad_head = int((head != GUARD_BYTE).sum())
        bad_tail = int((tail != GUARD_BYTE).sum())
        assert bad_head == 0 and bad_tail == 0, \
            f"{name}: {bad_head} guard bytes changed before and {bad_tail} after the buffer"


def run_gpu(q, k, v, causal, scale, k_len=None, out_dtype=torch.float32, flags=0, stream=None, num_splits=0,
            descale=(0.0, 0.0, 0.0)):
    """Run fa_fwd_ex on cuda:0; returns (O [B,H,N,d] fp32 CPU, lse [B,H,N] CPU).

    Outputs (and any split workspace) start as NaN so rows the kernels fail to
    write are caught, and sit between guard regions that must come back
    untouched.  num_splits = -1 takes the library's suggestion."""
    dev = torch.device("cuda:0")
    B, H, N, d = q.shape
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    kl = None if k_len is None else torch.as_tensor(k_len, dtype=torch.int32).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    og = Guarded((B, H, N, d), out_dtype, dev, fill=float("nan"))
    lg = Guarded((B, H, N), torch.float32, dev, fill=float("nan"))
    o, lse = og.t, lg.t
    if num_splits < 0:
        num_splits = fb.suggest_splits(qd, kd)
    wg, ws = None, None
    if num_splits > 1:
        nbytes = fb.workspace_bytes(qd, kd, num_splits)
        wg = Guarded((max(nbytes, 16) // 4,), torch.float32, dev, fill=float("nan"))
        ws = wg.t
    fb.fa_fwd_ex(qd, kd, vd, o, lse, causal, scale, k_len=kl, dev_status=status, flags=flags, stream=stream,
                 num_splits=num_splits, workspace=ws, descale=descale)
    st = fb.read_device_status(status, stream=stream)
    assert st == fb.FA_OK, fb.status_string(st)
    og.check("o")
    lg.check("lse")
    if wg is not None:
        wg.check("workspace")
    return o.float().cpu(), lse.cpu()


def compare(o_rows, lse_rows, o_ref, lse_ref, tol_max=TOL_MAX, tol_mean=TOL_MEAN, tol_lse=TOL_LSE):
    """Element-wise comparison of GPU rows with oracle rows; asserts and returns stats."""
    o_rows = np.asarray(o_rows, dtype=np.float64).reshape(o_ref.shape)
    lse_rows = np.asarray(lse_rows, dtype=np.float64).reshape(lse_ref.shape)
    empty = np.isneginf(lse_ref)
    assert np.all(np.isneginf(lse_rows[empty])), "rows with no allowed key must give lse = -inf"
    assert np.all(o_rows[empty] == 0.0), "rows with no allowed key must give O = 0"
    assert np.all(np.isfinite(o_rows)), "non-finite output"
    dO = np.abs(o_rows - o_ref)
    live = ~empty
    rel_lse = np.abs(lse_rows[live] - lse_ref[live]) / np.maximum(np.abs(lse_ref[live]), 1.0)
    stats = {"max_dO": float(dO.max()) if dO.size else 0.0, "mean_dO": float(dO.mean()) if dO.size else 0.0,
             "max_rel_lse": float(rel_lse.max()) if rel_lse.size else 0.0, "rows": int(lse_ref.size)}
    assert stats["max_dO"] <= tol_max, stats
    assert stats["mean_dO"] <= tol_mean, stats
    assert stats["max_rel_lse"] <= tol_lse, stats
    return stats


def check_case(q, k, v, causal, scale, k_len=None, rows=None, out_dtype=torch.float32, flags=0, num_splits=0,
               **tol):
    o, lse = run_gpu(q, k, v, causal, scale, k_len=k_len, out_dtype=out_dtype, flags=flags, num_splits=num_splits)
    B, H, N, d = q.shape
    o_ref, lse_ref = oracle.attention_f64(q, k, v, causal, scale, k_len=None if k_len is None else list(k_len),
                                          rows=rows)
    o_flat = o.reshape(-1, d).numpy()
    lse_flat = lse.reshape(-1).numpy()
    if rows is not None:
        o_flat, lse_flat = o_flat[rows], lse_flat[rows]
    return compare(o_flat, lse_flat, o_ref, lse_ref, **tol)


def check_workload(w: workloads.Workload, **kw):
    q, k, v, k_len = workloads.make_inputs(w)
    rows = None if w.sample_rows_per_head is None else workloads.sample_rows(w)
    kw.setdefault("num_splits", w.splits)
    return check_case(q, k, v, w.causal, w.scale, k_len=None if k_len is None else k_len.tolist(),
                      rows=rows, **kw)
