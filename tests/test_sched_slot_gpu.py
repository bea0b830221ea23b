"""The dynamic scheduler's launch slots: every causal launch (forward d = 64,
128, 256 and the backward) claims its slot for its own grid before it takes a
unit and frees it when its last CTA leaves.  A slot held by another launch is
waited for, bounded by the launch's time limit; when the limit passes the
launch does no work and reports FA_ERR_SCHED_BUSY.  The busy slot is made
with the library's test hook (the owner word written from the host, as an
in-flight launch would hold it), so no race between launches is needed."""
import ctypes
import math

import numpy as np
import pytest
import torch

from exact_io_aware_52_b200 import _binding as fb
from tests.gpu_util import check_case

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
FOREIGN = (0, 0, 0x5EED0001, 0x00000042)  # an owner no launch of this process has


def slot_words(slot):
    out = (ctypes.c_uint32 * 4)()
    assert fb.load().fa_testhook_sched_slot(slot, None, out) == fb.FA_OK
    return tuple(out)


def set_slot(slot, words):
    arr = (ctypes.c_uint32 * 4)(*words)
    assert fb.load().fa_testhook_sched_slot(slot, arr, None) == fb.FA_OK


def inputs(N, d, seed):
    g = torch.Generator().manual_seed(seed)
    return tuple(torch.randn(1, 2, N, d, generator=g).to(torch.bfloat16) for _ in range(3))


def test_hook_rejects_bad_slots():
    lib = fb.load()
    assert lib.fa_testhook_sched_slot(-1, None, None) == fb.FA_ERR_INVALID_ARGUMENT
    assert lib.fa_testhook_sched_slot(64, None, None) == fb.FA_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("d", [64, 128, 256])
def test_slot_is_free_after_each_causal_launch(d):
    q, k, v = inputs(700, d, seed=91 + d)
    slot = fb.load().fa_testhook_sched_next_slot()
    assert slot_words(slot) == (0, 0, 0, 0)
    check_case(q, k, v, True, 1.0 / math.sqrt(d))
    torch.cuda.synchronize()
    assert slot_words(slot) == (0, 0, 0, 0)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_forward_on_a_busy_slot_reports_and_does_nothing(d):
    q, k, v = inputs(700, d, seed=92 + d)
    qd, kd, vd = (t.to(DEV) for t in (q, k, v))
    o = torch.full((1, 2, 700, d), float("nan"), device=DEV)
    lse = torch.full((1, 2, 700), float("nan"), device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    slot = fb.load().fa_testhook_sched_next_slot()
    set_slot(slot, FOREIGN)
    try:
        fb.fa_fwd_ex(qd, kd, vd, o, lse, True, 1.0 / math.sqrt(d), dev_status=status, timeout_ms=20)
        assert fb.read_device_status(status) == fb.FA_ERR_SCHED_BUSY
        assert bool(torch.isnan(o).all()) and bool(torch.isnan(lse).all())  # no unit ran
        assert slot_words(slot) == FOREIGN  # the other launch's words are untouched
    finally:
        set_slot(slot, (0, 0, 0, 0))
    # the library is usable afterwards, and the freed slot serves the next launch on it
    check_case(q, k, v, True, 1.0 / math.sqrt(d))


def test_backward_on_a_busy_slot_reports_and_does_nothing():
    q, k, v = inputs(300, 128, seed=93)
    do = torch.randn(1, 2, 300, 128, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o = torch.zeros(1, 2, 300, 128, device=DEV)
    lse = torch.zeros(1, 2, 300, device=DEV)
    fb.fa_fwd_ex(qd, kd, vd, o, lse, True, 1.0 / math.sqrt(128))
    dq = torch.full(q.shape, float("nan"), device=DEV)
    dk = torch.full(k.shape, float("nan"), device=DEV)
    dv = torch.full(v.shape, float("nan"), device=DEV)
    ws = torch.empty(max(fb.bwd_workspace_bytes(qd), 16), dtype=torch.uint8, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    slot = fb.load().fa_testhook_sched_next_slot()
    set_slot(slot, FOREIGN)
    try:
        fb.fa_bwd(qd, kd, vd, o, lse, dod, dq, dk, dv, True, 1.0 / math.sqrt(128), ws, dev_status=status,
                  timeout_ms=20)
        assert fb.read_device_status(status) == fb.FA_ERR_SCHED_BUSY
        # the prep launch zeroes dq before the gradient kernel; dk and dv are never written
        assert bool((dq == 0).all()) and bool(torch.isnan(dk).all()) and bool(torch.isnan(dv).all())
        assert slot_words(slot) == FOREIGN
    finally:
        set_slot(slot, (0, 0, 0, 0))
    dq.fill_(float("nan"))
    status.zero_()
    fb.fa_bwd(qd, kd, vd, o, lse, dod, dq, dk, dv, True, 1.0 / math.sqrt(128), ws, dev_status=status)
    assert fb.read_device_status(status) == fb.FA_OK
    assert np.isfinite(dq.cpu().numpy()).all() and np.isfinite(dk.cpu().numpy()).all()
