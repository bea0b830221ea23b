"""Error bound of the E4M3 forward pass against the exact definition.

With E4M3 inputs the kernel computes Q K^T exactly up to fp32 accumulation
(a product of two E4M3 values has at most 8 significant bits), but rounds the
probabilities to E4M3 before the product with V.  It takes them relative to
a reference r minus 7 (log2 units) that trails the running row maximum by at
most tau (1.75, or 0 with eager rescaling): each weight 2^(7 + x_j - r) <=
2^8.75 < 448 is rounded either relatively (|dp| <= u p, u = 2^-4, three
mantissa bits, for weights >= 2^-6, E4M3's smallest normal) or absolutely
(|dp| <= 2^-10, half the subnormal spacing 2^-9, below it).  A weight taken
while the reference was smaller is only larger at rounding time and is then
scaled down exactly.  In units of the true row maximum m (p'_j = 2^(7 + x_j -
m)) the final reference lies delta, 0 <= delta <= tau, below m: the
absolutely rounded weights are a subset of those with p'_j < 2^-6, and their
error over the sum is at most 2^-10 / (2^delta L') <= 2^-10 / L'.  O is
divided by the unrounded sum, which is L' = sum_j p'_j in units of m, hence

    |O_kernel - O| = |sum_j dp_j v_j| / L'
                  <= u sum_j w_j |v_j| + 2^-10 / L' * sum_{j: p'_j < 2^-6} |v_j|

with w_j = p'_j / L' the exact softmax weights.  The test bound adds 10% to
the first term (exp2 approximation, fp32 accumulation) and 1e-4 absolute.
This module holds test arithmetic only; expected outputs come from the oracle.
"""
from __future__ import annotations

import numpy as np

U_E4M3 = 2.0 ** -4
SUB_E4M3 = 2.0 ** -6     # smallest normal
HALF_SUB_SPACING = 2.0 ** -10
SHIFT = 7.0


def bound_rows(q, k, v, causal: bool, scale: float, k_len=None, rows=None):
    """Per-element bound [n_rows, d] for flat row ids `rows` (all when None).

    q [B, H, N, d], k, v [B, H_kv, N_k, d]: float64 arrays of the values the
    kernel multiplies (dequantized); scale: the softmax scale applied to q.k."""
    B, H, N, d = q.shape
    H_kv, Nk = k.shape[1], k.shape[2]
    if rows is None:
        rows = np.arange(B * H * N)
    out = np.zeros((len(rows), d))
    log2e = 1.0 / np.log(2.0)
    for t, r in enumerate(rows):
        bh, i = divmod(int(r), N)
        b, h = divmod(bh, H)
        hk = h // (H // H_kv)
        lim = Nk if k_len is None else min(max(int(k_len[b]), 0), Nk)
        if causal:
            lim = min(lim, i + 1 + Nk - N)
        if lim <= 0:
            continue
        x = (k[b, hk, :lim] @ q[b, h, i]) * scale * log2e
        pp = np.exp2(SHIFT + x - x.max())
        L = pp.sum()
        w = pp / L
        va = np.abs(v[b, hk, :lim])
        sub = pp < SUB_E4M3
        out[t] = 1.1 * U_E4M3 * (w @ va) + HALF_SUB_SPACING / L * va[sub].sum(axis=0) + 1e-4
    return out
