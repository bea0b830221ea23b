"""fa_fwd_static_workspace: the key-split forward with its scratch in the
library's fixed device array.  Collected last (file name), so it runs both
alone and after every other test in one process.

It must give the result of fa_fwd_ex with a caller-owned workspace, on each
of two calls in a row, allocate no device memory across calls, and reject a
problem whose splits need more than the array holds."""
import math

import pytest
import torch

from exact_io_aware_52_b200 import _binding as fb
from tests.gpu_util import TOL_LSE, TOL_MAX, TOL_MEAN

pytestmark = pytest.mark.gpu


def _inputs(B, H, H_kv, Nq, Nk, d, seed):
    g = torch.Generator().manual_seed(seed)
    dev = torch.device("cuda:0")
    q = torch.randn(B, H, Nq, d, generator=g).to(torch.bfloat16).to(dev)
    k = torch.randn(B, H_kv, Nk, d, generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn(B, H_kv, Nk, d, generator=g).to(torch.bfloat16).to(dev)
    return q, k, v


def _close(o, lse, o_ref, lse_ref):
    dO = (o.float() - o_ref.float()).abs()
    assert torch.isfinite(o).all()
    assert dO.max().item() <= TOL_MAX and dO.mean().item() <= TOL_MEAN
    rel = (lse - lse_ref).abs() / lse_ref.abs().clamp_min(1.0)
    assert rel.max().item() <= TOL_LSE


@pytest.mark.parametrize("d,causal,splits", [(128, True, 9), (64, False, 4)])
def test_static_workspace_matches_caller_workspace(d, causal, splits):
    B, H, H_kv, Nq, Nk = 1, 8, 2, 256, 20000
    q, k, v = _inputs(B, H, H_kv, Nq, Nk, d, seed=90 + d)
    scale = 1.0 / math.sqrt(d)
    dev = q.device
    o_ref = torch.empty(B, H, Nq, d, device=dev)
    lse_ref = torch.empty(B, H, Nq, device=dev)
    ws = torch.empty(fb.workspace_bytes(q, k, splits), dtype=torch.uint8, device=dev)
    assert 0 < ws.numel() <= fb.FA_STATIC_WORKSPACE_BYTES
    fb.fa_fwd_ex(q, k, v, o_ref, lse_ref, causal, scale, num_splits=splits, workspace=ws)
    for call in range(2):  # two calls in a row on the same array
        o = torch.full((B, H, Nq, d), float("nan"), device=dev)
        lse = torch.full((B, H, Nq), float("nan"), device=dev)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        fb.fa_fwd_static_workspace(q, k, v, o, lse, causal, scale, dev_status=st, num_splits=splits)
        assert fb.read_device_status(st) == fb.FA_OK, call
        _close(o, lse, o_ref, lse_ref)


def test_static_workspace_allocates_nothing():
    q, k, v = _inputs(1, 4, 4, 128, 8192, 128, seed=93)
    dev = q.device
    o = torch.empty(1, 4, 128, 128, device=dev)
    lse = torch.empty(1, 4, 128, device=dev)
    fb.fa_fwd_static_workspace(q, k, v, o, lse, True, 0.088, num_splits=6)  # setup call
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        fb.fa_fwd_static_workspace(q, k, v, o, lse, True, 0.088, num_splits=6)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free0 == free1


def test_static_workspace_rejects_oversize_problem():
    # 16 splits x 8 x 1024 rows x (128 + 1) x 4 bytes = 67.6 MB > 64 MiB
    q, k, v = _inputs(1, 8, 8, 1024, 4096, 128, seed=94)
    assert fb.workspace_bytes(q, k, 16) > fb.FA_STATIC_WORKSPACE_BYTES
    o = torch.full((1, 8, 1024, 128), 7.0, device=q.device)
    lse = torch.full((1, 8, 1024), 7.0, device=q.device)
    with pytest.raises(fb.FaError) as e:
        fb.fa_fwd_static_workspace(q, k, v, o, lse, True, 0.088, num_splits=16)
    assert e.value.status == fb.FA_ERR_WORKSPACE_LIMIT
    torch.cuda.synchronize()
    assert (o == 7.0).all() and (lse == 7.0).all()  # nothing was launched
