"""The E4M3 error bound (tests/fp8_bound.py) holds for the rounding it
describes: probabilities taken relative to a reference up to tau below the row
maximum, minus the shift, rounded to E4M3 by torch, O divided by the
unrounded sum.  Checked against the fp64 oracle on random and peaked rows,
with the reference at the maximum and lagging it, where it must also not be
vacuous."""
import math

import numpy as np
import torch

import oracle
from tests import fp8_bound


TAU = 1.75  # the kernel's rescale threshold for E4M3 inputs (log2 units)


def _emulate(q, k, v, scale, lag=None):
    """O of the rounding model: weights 2^(SHIFT + x - r) rounded to E4M3, with
    the reference r = max - lag (lag per row in [0, TAU]; 0 when None)."""
    x = torch.einsum("bhid,bhjd->bhij", q, k) * scale / math.log(2.0)
    r = x.amax(-1, keepdim=True)
    if lag is not None:
        r = r - lag
    pp = torch.exp2(fp8_bound.SHIFT + x - r)
    assert pp.max().item() <= 2.0 ** (fp8_bound.SHIFT + TAU) < 448.0
    pr = pp.float().to(torch.float8_e4m3fn).double()
    return torch.einsum("bhij,bhjd->bhid", pr, v) / pp.sum(-1, keepdim=True)


def test_bound_holds_for_the_rounding_model():
    g = torch.Generator().manual_seed(7)
    for std in (1.0, 3.0):
        q = (torch.randn(1, 2, 64, 128, generator=g) * std).to(torch.float8_e4m3fn)
        k = (torch.randn(1, 2, 200, 128, generator=g) * std).to(torch.float8_e4m3fn)
        v = torch.randn(1, 2, 200, 128, generator=g).to(torch.float8_e4m3fn)
        scale = float(np.float32(1 / math.sqrt(128)))
        o_ref, _ = oracle.attention_f64(q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16), False,
                                        scale)
        bound = fp8_bound.bound_rows(q.double().numpy(), k.double().numpy(), v.double().numpy(), False, scale)
        lag = torch.rand(1, 2, 64, 1, generator=g, dtype=torch.float64) * TAU
        for lg in (None, lag):
            o_emul = _emulate(q.double(), k.double(), v.double(), scale, lg).numpy().reshape(o_ref.shape)
            err = np.abs(o_emul - o_ref)
            assert np.all(err <= bound)
            assert err.max() > 0.05 * bound.max()  # the bound is not vacuously loose here
