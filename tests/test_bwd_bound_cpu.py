"""The backward error bound (tests/bwd_bound.py) holds for the rounding it
describes -- P and dS rounded to bf16 -- against the fp64 backward oracle,
and is not vacuous."""
import math

import numpy as np
import torch

import oracle
from tests import bwd_bound


def _bf16(x):
    return torch.from_numpy(x).to(torch.bfloat16).double().numpy()


def test_bound_holds_for_the_rounding_model():
    g = torch.Generator().manual_seed(9)
    B, H, H_kv, N, Nk, d = 1, 4, 2, 48, 80, 32
    for causal, std in ((False, 1.0), (True, 2.5)):
        q = (torch.randn(B, H, N, d, generator=g) * std).to(torch.bfloat16)
        k = (torch.randn(B, H_kv, Nk, d, generator=g) * std).to(torch.bfloat16)
        v = torch.randn(B, H_kv, Nk, d, generator=g).to(torch.bfloat16)
        do = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
        scale = float(np.float32(1 / math.sqrt(d)))
        dq, dk, dv = oracle.attention_bwd_f64(q, k, v, do, causal, scale)
        qd, kd, vd, dod = (t.double().numpy() for t in (q, k, v, do))
        # the rounding model, in float64 otherwise
        eq, ek, ev = np.zeros_like(dq), np.zeros_like(dk), np.zeros_like(dv)
        for h in range(H):
            hk = h // (H // H_kv)
            s = scale * qd[0, h] @ kd[0, hk].T
            if causal:
                s = np.where(np.arange(Nk)[None, :] <= np.arange(N)[:, None] + Nk - N, s, -np.inf)
            P = np.exp(s - s.max(1, keepdims=True))
            P /= P.sum(1, keepdims=True)
            O = P @ vd[0, hk]
            Pr = _bf16(P)
            dS = _bf16(scale * Pr * (dod[0, h] @ vd[0, hk].T - (dod[0, h] * O).sum(1, keepdims=True)))
            ev[0, hk] += Pr.T @ dod[0, h]
            eq[0, h] = dS @ kd[0, hk]
            ek[0, hk] += dS.T @ qd[0, h]
        bq, bk, bv = bwd_bound.bounds(qd, kd, vd, dod, causal, scale)
        for name, emul, ref, bnd in (("dq", eq, dq, bq), ("dk", ek, dk, bk), ("dv", ev, dv, bv)):
            err = np.abs(emul - ref)
            assert np.all(err <= bnd), name
            assert err.max() > 0.02 * bnd.max(), name  # not vacuously loose


def test_row_chunks_give_the_same_bound():
    """Taking the query rows in chunks changes nothing but the order of the dK
    and dV bound sums (every other quantity of a row depends on that row)."""
    g = torch.Generator().manual_seed(10)
    B, H, H_kv, N, Nk, d = 2, 2, 1, 37, 50, 16
    q, do = (torch.randn(B, H, N, d, generator=g).double().numpy() for _ in range(2))
    k, v = (torch.randn(B, H_kv, Nk, d, generator=g).double().numpy() for _ in range(2))
    for causal in (False, True):
        whole = bwd_bound.bounds(q, k, v, do, causal, 0.25, k_len=[50, 20], row_chunk=N)
        for chunk in (1, 5, 16):
            part = bwd_bound.bounds(q, k, v, do, causal, 0.25, k_len=[50, 20], row_chunk=chunk)
            for a, b in zip(whole, part):
                np.testing.assert_allclose(a, b, rtol=1e-12, atol=0)
