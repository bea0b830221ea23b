"""Pins for the fp64 oracle: checks against facts that do not come from the
oracle itself.  Each pin takes an oracle library handle so that the same
checks also run against deliberately broken builds of the oracle source
(``test_oracle_mutants.py``), proving that each plausible mistake is caught.

Sources of truth used here, none of which is the oracle's own code:
* closed forms of special cases of softmax(Q K^T * scale) V (page
  "FlashAttention (ES)", section "El problema de la atencion estandar");
* invariants of the definition (permutation of keys, convexity, rows of the
  softmax summing to one, the softmax ratio property);
* library routines: torch's float64 scaled_dot_product_attention and
  logsumexp, scipy's logsumexp;
* brute force: the pure-Python online-softmax recurrence of section
  "Calculo de Softmax en linea" over every block size on tiny inputs.
"""
from __future__ import annotations

import itertools
import math

import numpy as np
import torch

import oracle
from oracle.online import attention_online


def bf16(x) -> torch.Tensor:
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def run(lib, q, k, v, causal, scale, k_len=None, rows=None):
    B, H, N, d = q.shape
    o, lse = oracle.attention_f64(q, k, v, causal, scale, k_len=k_len, rows=rows, lib=lib, nthreads=2)
    if rows is None:
        return o.reshape(B, H, N, d), lse.reshape(B, H, N)
    return o, lse


def allowed_end(i, N, causal, L):
    e = N if L is None else max(0, min(N, L))
    if causal:
        e = min(e, i + 1)
    return e


# ---------------------------------------------------------------------------
def pin_zero_query_means(lib):
    """Q = 0 gives equal weights: O_i is the mean of the allowed V rows and
    lse_i = ln(#allowed); no allowed key gives O = 0, lse = -inf."""
    g = torch.Generator().manual_seed(11)
    B, H, N, d = 2, 2, 37, 8
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
    k = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    vv = f64(v)
    for causal, k_len in itertools.product([False, True], [None, [5, 37], [0, 20]]):
        o, lse = run(lib, q, k, v, causal, 0.25, k_len=k_len)
        for b, h, i in itertools.product(range(B), range(H), range(N)):
            e = allowed_end(i, N, causal, None if k_len is None else k_len[b])
            if e == 0:
                assert np.all(o[b, h, i] == 0.0), (causal, k_len, b, h, i)
                assert lse[b, h, i] == -math.inf
                continue
            np.testing.assert_allclose(o[b, h, i], vv[b, h, :e].mean(axis=0), rtol=0, atol=1e-12)
            assert abs(lse[b, h, i] - math.log(e)) < 1e-12, (causal, k_len, b, h, i)


def pin_dominant_key(lib):
    """q_i = c e_{i mod d}, k_j = c e_{(j+1) mod d}: the score is
    delta = scale c^2 on keys with (j+1) = i (mod d) and 0 elsewhere, so
    O_i = (e^delta sum_{j in D} v_j + sum_{j not in D} v_j) / (e^delta |D| + n - |D|)
    over the n allowed keys.  Asymmetric, so a transposed Q K^T is caught."""
    g = torch.Generator().manual_seed(12)
    N, d, c, scale = 11, 4, 4.0, 0.5
    delta = scale * c * c
    qn = np.zeros((1, 1, N, d)); kn = np.zeros((1, 1, N, d))
    for i in range(N):
        qn[0, 0, i, i % d] = c
        kn[0, 0, i, (i + 1) % d] = c
    q, k = bf16(qn), bf16(kn)
    v = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    vv = f64(v)[0, 0]
    for causal in (False, True):
        o, lse = run(lib, q, k, v, causal, scale)
        for i in range(N):
            n = allowed_end(i, N, causal, None)
            D = [j for j in range(n) if (j + 1) % d == i % d]
            w = np.array([math.exp(delta) if j in D else 1.0 for j in range(n)])
            ref = (w[:, None] * vv[:n]).sum(0) / w.sum()
            np.testing.assert_allclose(o[0, 0, i], ref, rtol=1e-13, atol=1e-13)
            assert abs(lse[0, 0, i] - math.log(w.sum())) < 1e-12


def _sdpa_ref(q, k, v, causal, scale, k_len):
    scale = float(np.float32(scale))  # the oracle takes the float32 value of the scale
    qd, kd, vd = (t.to(torch.float64) for t in (q, k, v))
    B, H, N, d = q.shape
    mask = torch.ones(B, 1, N, N, dtype=torch.bool)
    if causal:
        mask &= torch.ones(N, N, dtype=torch.bool).tril()
    if k_len is not None:
        for b in range(B):
            mask[b, :, :, k_len[b]:] = False
    o = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, attn_mask=mask, scale=scale)
    s = (qd @ kd.transpose(-1, -2)) * scale
    s = s.masked_fill(~mask, -math.inf)
    return o.numpy(), torch.logsumexp(s, dim=-1).numpy()


def pin_library_sdpa(lib):
    """Random inputs against torch's float64 scaled_dot_product_attention and
    logsumexp (causal, key padding, several logit scales)."""
    g = torch.Generator().manual_seed(13)
    B, H, N, d = 2, 3, 45, 16
    for std, causal, k_len in itertools.product([1.0, 3.0], [False, True], [None, [7, 45]]):
        q = (torch.randn(B, H, N, d, generator=g) * std).to(torch.bfloat16)
        k = (torch.randn(B, H, N, d, generator=g) * std).to(torch.bfloat16)
        v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
        scale = 1.0 / math.sqrt(d) * 0.9
        o, lse = run(lib, q, k, v, causal, scale, k_len=k_len)
        o_ref, lse_ref = _sdpa_ref(q, k, v, causal, scale, k_len)
        np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def pin_permutation_invariance(lib):
    """Non-causal attention does not depend on the order of the key/value
    pairs: permuting K and V rows together leaves O and lse unchanged."""
    g = torch.Generator().manual_seed(14)
    B, H, N, d = 1, 2, 33, 8
    q = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    perm = torch.randperm(N, generator=g)
    o1, l1 = run(lib, q, k, v, False, 0.3)
    o2, l2 = run(lib, q, k[:, :, perm], v[:, :, perm], False, 0.3)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)
    # a permutation of the queries permutes the outputs
    o3, l3 = run(lib, q[:, :, perm], k, v, False, 0.3)
    np.testing.assert_allclose(o3, o1[:, :, perm.numpy()], rtol=0, atol=1e-15)
    np.testing.assert_allclose(l3, l1[:, :, perm.numpy()], rtol=0, atol=1e-15)


def pin_single_key(lib):
    """N = 1: the only key gets weight 1, so O = V_0 and lse = scale q_0.k_0."""
    g = torch.Generator().manual_seed(15)
    for causal in (False, True):
        q = torch.randn(2, 2, 1, 8, generator=g).to(torch.bfloat16)
        k = torch.randn(2, 2, 1, 8, generator=g).to(torch.bfloat16)
        v = torch.randn(2, 2, 1, 8, generator=g).to(torch.bfloat16)
        o, lse = run(lib, q, k, v, causal, 0.7)
        np.testing.assert_array_equal(o, f64(v))
        s = (f64(q) * f64(k)).sum(-1) * float(np.float32(0.7))
        np.testing.assert_allclose(lse, s, rtol=0, atol=1e-14)


def pin_constant_values(lib):
    """Constant V rows give that constant for every row with an allowed key."""
    g = torch.Generator().manual_seed(16)
    B, H, N, d = 2, 1, 29, 8
    q = (torch.randn(B, H, N, d, generator=g) * 2).to(torch.bfloat16)
    k = (torch.randn(B, H, N, d, generator=g) * 2).to(torch.bfloat16)
    v = torch.full((B, H, N, d), -1.75).to(torch.bfloat16)
    for causal, k_len in itertools.product([False, True], [None, [3, 29]]):
        o, _ = run(lib, q, k, v, causal, 0.4, k_len=k_len)
        np.testing.assert_allclose(o, -1.75, rtol=0, atol=1e-14)


def pin_rows_are_distributions(lib):
    """With V = identity (N = d) each output row IS the softmax row: entries are
    >= 0, masked entries exactly 0, rows sum to 1, and every ratio
    P_ij / P_ik equals exp(s_ij - s_ik) with s = scale q.k from numpy."""
    g = torch.Generator().manual_seed(17)
    N = d = 16
    q = torch.randn(1, 2, N, d, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 2, N, d, generator=g).to(torch.bfloat16)
    v = torch.eye(N).expand(1, 2, N, N).contiguous().to(torch.bfloat16)
    scale = 0.6
    s = np.einsum("bhid,bhjd->bhij", f64(q), f64(k)) * float(np.float32(scale))
    for causal, L in itertools.product([False, True], [None, 9]):
        P, _ = run(lib, q, k, v, causal, scale, k_len=None if L is None else [L])
        for h, i in itertools.product(range(2), range(N)):
            e = allowed_end(i, N, causal, L)
            row = P[0, h, i]
            assert np.all(row >= 0)
            assert np.all(row[e:] == 0.0)
            assert abs(row.sum() - 1.0) < 1e-13
            for j in range(1, e):
                assert abs(math.log(row[j] / row[0]) - (s[0, h, i, j] - s[0, h, i, 0])) < 1e-11


def pin_convex_hull(lib):
    """Each output is a convex combination of the allowed V rows, so every
    column lies within [min, max] of that column over the allowed rows."""
    g = torch.Generator().manual_seed(18)
    B, H, N, d = 1, 2, 40, 8
    q = (torch.randn(B, H, N, d, generator=g) * 3).to(torch.bfloat16)
    k = (torch.randn(B, H, N, d, generator=g) * 3).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    vv = f64(v)
    o, _ = run(lib, q, k, v, True, 0.5, k_len=[31])
    for h, i in itertools.product(range(H), range(N)):
        e = allowed_end(i, N, True, 31)
        lo, hi = vv[0, h, :e].min(0), vv[0, h, :e].max(0)
        assert np.all(o[0, h, i] >= lo - 1e-13) and np.all(o[0, h, i] <= hi + 1e-13)


def pin_online_equals_two_pass(lib):
    """The block-wise online-softmax recurrence, run with every block size on
    brute-forced tiny inputs (ties, masked rows, fully masked blocks),
    equals the two-pass definition."""
    rng = np.random.default_rng(19)
    cases = 0
    for N, d in [(1, 1), (2, 1), (3, 2), (5, 2), (8, 4)]:
        for causal in (False, True):
            for L in sorted({0, 1, max(N - 1, 0), N}):
                # small integers make ties between scores common
                qn = rng.integers(-2, 3, size=(1, 2, N, d)).astype(np.float64)
                kn = rng.integers(-2, 3, size=(1, 2, N, d)).astype(np.float64)
                vn = rng.integers(-4, 5, size=(1, 2, N, d)).astype(np.float64) / 4
                q, k, v = bf16(qn), bf16(kn), bf16(vn)
                o_ref, lse_ref = run(lib, q, k, v, causal, 0.75, k_len=[L])
                for tile in range(1, N + 1):
                    o_on, lse_on = attention_online(f64(q), f64(k), f64(v), causal, float(np.float32(0.75)),
                                                    k_len=[L], tile=tile)
                    np.testing.assert_allclose(np.array(o_on), o_ref, rtol=0, atol=1e-13)
                    np.testing.assert_allclose(np.array(lse_on), lse_ref, rtol=0, atol=1e-13)
                    cases += 1
    assert cases > 50


def pin_large_logits(lib):
    """Scores near +-1e3 overflow exp() unless the maximum is subtracted:
    lse against scipy's logsumexp of numpy scores, O against torch's fp64
    scaled_dot_product_attention."""
    from scipy.special import logsumexp

    g = torch.Generator().manual_seed(20)
    B, H, N, d = 1, 2, 24, 4
    q = (torch.randn(B, H, N, d, generator=g) * 30).to(torch.bfloat16)
    k = (torch.randn(B, H, N, d, generator=g) * 30).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    scale = 0.5
    for causal in (False, True):
        o, lse = run(lib, q, k, v, causal, scale)
        s = np.einsum("bhid,bhjd->bhij", f64(q), f64(k)) * scale
        assert np.abs(s).max() > 750  # exp would overflow without the max shift
        for h, i in itertools.product(range(H), range(N)):
            e = allowed_end(i, N, causal, None)
            assert abs(lse[0, h, i] - logsumexp(s[0, h, i, :e])) <= 1e-12 * max(1.0, abs(lse[0, h, i]))
        o_ref, _ = _sdpa_ref(q, k, v, causal, scale, None)
        np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-11)


def pin_row_subset(lib):
    """Asking for a subset of rows returns exactly those rows of the full result."""
    g = torch.Generator().manual_seed(21)
    B, H, N, d = 2, 2, 19, 8
    q = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    o, lse = run(lib, q, k, v, True, 0.3, k_len=[10, 19])
    rows = np.array([0, 5, 18, 19, 40, 75], dtype=np.int64)
    o_s, lse_s = run(lib, q, k, v, True, 0.3, k_len=[10, 19], rows=rows)
    np.testing.assert_array_equal(o_s, o.reshape(-1, d)[rows])
    np.testing.assert_array_equal(lse_s, lse.reshape(-1)[rows])


def pin_grouped_heads(lib):
    """Grouped key/value heads: against torch's float64 scaled_dot_product_attention
    with enable_gqa (a library routine), and equal to multi-head attention on K, V
    with each key/value head repeated H / H_kv times; H_kv = 1 is multi-query."""
    g = torch.Generator().manual_seed(22)
    B, H, N, d = 2, 6, 23, 8
    for H_kv in (1, 2, 3):
        q = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
        k = torch.randn(B, H_kv, N, d, generator=g).to(torch.bfloat16)
        v = torch.randn(B, H_kv, N, d, generator=g).to(torch.bfloat16)
        for causal, k_len in ((False, None), (True, [20, 9])):
            o, lse = run(lib, q, k, v, causal, 0.35, k_len=k_len)
            rep = H // H_kv
            o_mha, lse_mha = run(lib, q, k.repeat_interleave(rep, dim=1), v.repeat_interleave(rep, dim=1),
                                 causal, 0.35, k_len=k_len)
            np.testing.assert_array_equal(o, o_mha)
            np.testing.assert_array_equal(lse, lse_mha)
            scale = float(np.float32(0.35))
            mask = torch.ones(B, 1, N, N, dtype=torch.bool)
            if causal:
                mask &= torch.ones(N, N, dtype=torch.bool).tril()
            if k_len is not None:
                for b in range(B):
                    mask[b, :, :, k_len[b]:] = False
            o_ref = torch.nn.functional.scaled_dot_product_attention(
                q.double(), k.double(), v.double(), attn_mask=mask, scale=scale, enable_gqa=True)
            np.testing.assert_allclose(o, o_ref.numpy(), rtol=1e-10, atol=1e-11)


def pin_fewer_queries_than_keys(lib):
    """N_q queries against N_k > N_q keys: against torch's float64
    scaled_dot_product_attention with the bottom-right causal mask (key j
    allowed for query i iff j <= i + N_k - N_q), and equal to the last N_q
    rows of the square problem whose last N_q query rows are these queries."""
    g = torch.Generator().manual_seed(23)
    B, H, Nq, Nk, d = 2, 2, 7, 30, 8
    q = torch.randn(B, H, Nq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, H, Nk, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, Nk, d, generator=g).to(torch.bfloat16)
    scale = float(np.float32(0.4))
    for causal, k_len in ((False, None), (True, None), (True, [27, 30])):
        o, lse = run(lib, q, k, v, causal, 0.4, k_len=k_len)
        mask = torch.ones(B, 1, Nq, Nk, dtype=torch.bool)
        if causal:
            mask &= torch.ones(Nq, Nk, dtype=torch.bool).tril(diagonal=Nk - Nq)
        if k_len is not None:
            for b in range(B):
                mask[b, :, :, k_len[b]:] = False
        o_ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double(),
                                                                 attn_mask=mask, scale=scale)
        np.testing.assert_allclose(o, o_ref.numpy(), rtol=1e-10, atol=1e-11)
        qfull = torch.randn(B, H, Nk, d, generator=g).to(torch.bfloat16)
        qfull[:, :, Nk - Nq:] = q
        o_sq, lse_sq = run(lib, qfull, k, v, causal, 0.4, k_len=k_len)
        np.testing.assert_array_equal(o, o_sq[:, :, Nk - Nq:])
        np.testing.assert_array_equal(lse, lse_sq[:, :, Nk - Nq:])


ALL_PINS = [pin_zero_query_means, pin_dominant_key, pin_library_sdpa, pin_permutation_invariance,
            pin_single_key, pin_constant_values, pin_rows_are_distributions, pin_convex_hull,
            pin_online_equals_two_pass, pin_large_logits, pin_row_subset, pin_grouped_heads,
            pin_fewer_queries_than_keys]
