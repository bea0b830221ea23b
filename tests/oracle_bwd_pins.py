"""Pins for the fp64 backward oracle (attn_bwd_oracle.c): checks against facts
that do not come from the backward oracle itself.  Each pin takes a backward
library handle so that the same checks run against deliberately broken builds
(``test_bwd_pins_catch_mutant`` in ``test_oracle_bwd.py``).

Sources of truth:
* a library routine: torch's float64 autograd through scaled_dot_product_attention
  (with explicit masks for causal, bottom-right and key padding, and
  ``enable_gqa`` for grouped heads);
* finite differences of the (separately pinned) forward oracle: central
  differences of L = sum(O * dO) with bf16-exact steps;
* closed forms and invariants of the derivative: one key gives dQ = dK = 0
  and dV = sum of dO; every row of dS sums to zero, so dK sums to zero over
  the keys; the rows of P sum to one, so dV sums to the sum of dO over rows
  that have an allowed key; the gradients are linear in dO.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


def _bwd(lib, q, k, v, do, causal, scale, k_len=None):
    return oracle.attention_bwd_f64(q, k, v, do, causal, scale, k_len=k_len, lib=lib, nthreads=2)


def _rand(shape, g, std=1.0):
    return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16)


def _mask(N, Nk, causal, L):
    m = torch.ones(N, Nk, dtype=torch.bool)
    if causal:
        m = m.tril(diagonal=Nk - N)
    if L is not None:
        m[:, max(0, min(Nk, L)):] = False
    return m


def _autograd(q, k, v, do, causal, scale, k_len=None):
    B, H, N, d = q.shape
    H_kv, Nk = k.shape[1], k.shape[2]
    Q, K, V = (t.double().requires_grad_() for t in (q, k, v))
    s32 = float(np.float32(scale))
    outs = []
    for b in range(B):
        L = None if k_len is None else int(k_len[b])
        m = _mask(N, Nk, causal, L)
        o = torch.nn.functional.scaled_dot_product_attention(Q[b:b + 1], K[b:b + 1], V[b:b + 1], attn_mask=m,
                                                             scale=s32, enable_gqa=H_kv != H)
        # rows with no allowed key: SDPA gives NaN; the definition gives O = 0 and no gradient
        empty = ~m.any(-1)
        o = torch.where(empty[None, None, :, None], torch.zeros_like(o), o)
        outs.append(o)
    O = torch.cat(outs, 0)
    O.backward(do.double())
    return Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()


def pin_autograd_sdpa(lib):
    """Gradients equal torch fp64 autograd through SDPA: square causal and
    non-causal, fewer queries than keys (bottom-right), key padding with an
    empty batch, grouped heads."""
    g = torch.Generator().manual_seed(501)
    cases = [
        dict(B=2, H=2, H_kv=2, N=9, Nk=9, d=8, causal=False, k_len=None),
        dict(B=2, H=2, H_kv=2, N=9, Nk=9, d=8, causal=True, k_len=None),
        dict(B=1, H=2, H_kv=2, N=5, Nk=12, d=8, causal=True, k_len=None),
        dict(B=3, H=1, H_kv=1, N=7, Nk=7, d=4, causal=True, k_len=[7, 3, 0]),
        dict(B=1, H=4, H_kv=2, N=6, Nk=6, d=8, causal=True, k_len=None),
        dict(B=1, H=3, H_kv=1, N=6, Nk=10, d=4, causal=False, k_len=[8]),
    ]
    for c in cases:
        q = _rand((c["B"], c["H"], c["N"], c["d"]), g)
        k = _rand((c["B"], c["H_kv"], c["Nk"], c["d"]), g)
        v = _rand((c["B"], c["H_kv"], c["Nk"], c["d"]), g)
        do = _rand((c["B"], c["H"], c["N"], c["d"]), g)
        scale = 0.4
        got = _bwd(lib, q, k, v, do, c["causal"], scale, c["k_len"])
        ref = _autograd(q, k, v, do, c["causal"], scale, c["k_len"])
        for name, a, b in zip(("dq", "dk", "dv"), got, ref):
            np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12, err_msg=f"{name} {c}")


def pin_finite_differences(lib):
    """Central differences of L = sum(O * dO) through the forward oracle, with
    inputs on a 2^-4 grid and steps of 2^-6 (both exact in bf16)."""
    g = torch.Generator().manual_seed(502)
    B, H, N, Nk, d = 1, 1, 4, 6, 3
    grid = lambda shape: (torch.randint(-24, 25, shape, generator=g).float() / 16).to(torch.bfloat16)  # noqa: E731
    q, k, v, do = grid((B, H, N, d)), grid((B, H, Nk, d)), grid((B, H, Nk, d)), grid((B, H, N, d))
    scale, h = 0.5, 2.0 ** -6
    dq, dk, dv = _bwd(lib, q, k, v, do, True, scale)
    dof = do.double().numpy()

    def loss(qq, kk, vv):
        o, _ = oracle.attention_f64(qq, kk, vv, True, scale, nthreads=1)
        return float((o.reshape(B, H, N, d) * dof).sum())

    for name, t, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in np.ndindex(*t.shape):
            tp, tm = t.clone(), t.clone()
            tp[idx] = (t[idx].float() + h).to(torch.bfloat16)
            tm[idx] = (t[idx].float() - h).to(torch.bfloat16)
            assert float(tp[idx]) - float(tm[idx]) == 2 * h
            args_p = {"q": (tp, k, v), "k": (q, tp, v), "v": (q, k, tp)}[name]
            args_m = {"q": (tm, k, v), "k": (q, tm, v), "v": (q, k, tm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - grad[idx]) <= 2e-3 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def pin_single_key(lib):
    """One allowed key: P = 1, so dS = 0 (dQ = dK = 0) and dV = sum_i dO_i."""
    g = torch.Generator().manual_seed(503)
    q, k, v, do = _rand((1, 2, 6, 8), g), _rand((1, 2, 1, 8), g), _rand((1, 2, 1, 8), g), _rand((1, 2, 6, 8), g)
    dq, dk, dv = _bwd(lib, q, k, v, do, False, 0.3)
    assert np.abs(dq).max() < 1e-12 and np.abs(dk).max() < 1e-12
    np.testing.assert_allclose(dv[:, :, 0], do.double().numpy().sum(2), rtol=1e-12, atol=1e-12)


def pin_row_sums(lib):
    """Every row of dS sums to zero, so dK sums to zero over the keys; the rows
    of P sum to one, so dV sums to the sum of dO over rows with an allowed key
    (here the causal rows and a padded batch with no key)."""
    g = torch.Generator().manual_seed(504)
    B, H, N, d = 2, 2, 11, 8
    q, k, v, do = (_rand((B, H, N, d), g) for _ in range(4))
    dq, dk, dv = _bwd(lib, q, k, v, do, True, 0.35, k_len=[11, 0])
    assert np.abs(dk.sum(2)).max() < 1e-10
    expect = do.double().numpy().sum(2)
    expect[1] = 0.0
    np.testing.assert_allclose(dv.sum(2), expect, rtol=1e-10, atol=1e-10)
    assert np.abs(dq[1]).max() == 0.0


def pin_equal_keys(lib):
    """Equal keys give equal scores in a row: dQ = sigma * k * sum_j dS_ij = 0."""
    g = torch.Generator().manual_seed(505)
    q, v, do = _rand((1, 1, 8, 8), g), _rand((1, 1, 8, 8), g), _rand((1, 1, 8, 8), g)
    k = _rand((1, 1, 1, 8), g).expand(1, 1, 8, 8).contiguous()
    dq, _, _ = _bwd(lib, q, k, v, do, True, 0.5)
    assert np.abs(dq).max() < 1e-12


def pin_linear_in_dout(lib):
    """The gradients are linear in dO (2 dO is exact in bf16)."""
    g = torch.Generator().manual_seed(506)
    q, k, v, do = (_rand((1, 2, 7, 8), g) for _ in range(4))
    a = _bwd(lib, q, k, v, do, True, 0.5)
    b = _bwd(lib, q, k, v, (do.float() * 2).to(torch.bfloat16), True, 0.5)
    for x, y in zip(a, b):
        np.testing.assert_allclose(2 * x, y, rtol=1e-12, atol=1e-14)


ALL_BWD_PINS = [pin_autograd_sdpa, pin_finite_differences, pin_single_key, pin_row_sums, pin_equal_keys,
                pin_linear_in_dout]
