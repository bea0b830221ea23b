"""The production forward kernels' time-out path, made to run for real.

With the test-only field `test_drop_load` the first CTA's TMA producer never
issues one chosen key-tile load (and never arms its barrier), so no copy is
ever in flight toward it: the MMA issuer's bounded wait for that tile runs out
after `timeout_ms`, the CTA raises its abort flag, every role leaves its loop,
the softmax warps mark the abandoned unit's rows NaN, the producer drains the
copies it did issue, TMEM is freed and the launch ends.  Nothing here faults,
traps or hangs the GPU: the wait is bounded and the status word reports it.

Checked: the call returns; the status word holds FA_ERR_DEVICE_TIMEOUT; the
abandoned unit's rows are NaN in O and lse; the other CTA's unit matches the
fp64 oracle; and the next normal launch in the same process is bit-identical
to a clean launch made before the time-out (which itself matches the oracle).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_52_b200 import _binding as fb
from tests.gpu_util import compare

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def launch(qd, kd, vd, causal, scale, d, **kw):
    o = torch.full(tuple(qd.shape), float("nan"), device=DEV)
    lse = torch.full(tuple(qd.shape[:3]), float("nan"), device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    fb.fa_fwd_ex(qd, kd, vd, o, lse, causal, scale, dev_status=st, **kw)
    return o, lse, fb.read_device_status(st)


@pytest.mark.parametrize("d,causal,dtype", [(64, False, "bf16"), (64, True, "bf16"), (128, False, "bf16"),
                                            (128, True, "bf16"), (128, False, "e4m3"), (256, False, "bf16"),
                                            (256, True, "bf16")])
def test_dropped_tile_times_out_cleanly(d, causal, dtype):
    N = 512
    g = torch.Generator().manual_seed(610 + d + causal)
    q, k, v = (torch.randn(1, 1, N, d, generator=g) for _ in range(3))
    dt = torch.float8_e4m3fn if dtype == "e4m3" else torch.bfloat16
    q, k, v = q.to(dt), k.to(dt), v.to(dt)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    scale = 1.0 / math.sqrt(d)

    o_ref_gpu, lse_ref_gpu, st = launch(qd, kd, vd, causal, scale, d)
    assert st == fb.FA_OK
    o_bad, lse_bad, st = launch(qd, kd, vd, causal, scale, d, timeout_ms=50, test_drop_load=1)
    assert st == fb.FA_ERR_DEVICE_TIMEOUT, fb.status_string(st)
    o_next, lse_next, st = launch(qd, kd, vd, causal, scale, d)
    assert st == fb.FA_OK

    # the first CTA's first unit is the last query block of head 0 (units are
    # numbered longest block first): 256 rows for d <= 128, 128 for d = 256
    rows = 128 if d == 256 else 256
    lost = slice(N - rows, N)
    kept = slice(0, N - rows)
    assert bool(torch.isnan(o_bad[0, 0, lost]).all()) and bool(torch.isnan(lse_bad[0, 0, lost]).all())

    qo, ko, vo = (t.to(torch.bfloat16) for t in (q, k, v))  # E4M3 widens exactly to bf16
    o_ref, lse_ref = oracle.attention_f64(qo, ko, vo, causal, scale)
    o_ref = o_ref.reshape(N, d)
    if dtype == "bf16":
        # the unit the other CTA ran is right despite the abandoned one
        compare(o_bad[0, 0, kept].cpu().numpy(), lse_bad[0, 0, kept].cpu().numpy(), o_ref[kept], lse_ref[kept])
        compare(o_ref_gpu[0, 0].cpu().numpy(), lse_ref_gpu[0, 0].cpu().numpy(), o_ref, lse_ref)
    else:
        assert torch.equal(o_bad[0, 0, kept], o_ref_gpu[0, 0, kept])
    # the next launch is unaffected: bit-identical to the clean one before
    assert torch.equal(o_next, o_ref_gpu) and torch.equal(lse_next, lse_ref_gpu)
    assert np.isfinite(o_next.cpu().numpy()).all()
