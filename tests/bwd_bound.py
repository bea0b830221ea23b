"""Error bound of the backward kernels against the exact gradients.

The kernels recompute P from Q, K and the forward's lse in fp32 and round it
to bf16 (unit roundoff u = 2^-8: 8 significant bits) for dV = P^T dO and for dS; they round
dS = sigma P (dP - D) to bf16 for dK = dS^T Q and dQ = dS K; every product
accumulates in fp32.  With the exact P, dP = dO V^T, D_i = dO_i . O_i and
dS, and e ~ 2e-5 covering the fp32 sums (dP, D, the tensor-core
accumulation, exp2 and the atomic fp32 additions into dQ):

    |dP~_ij - P_ij| <= (u + e) P_ij
    |dS~_ij - dS_ij| <= (2u + e) |dS_ij| + sigma P_ij e (|dO_i| |V_j| + |dO_i| |O_i|)  =: E_ij
    |dV~ - dV| <= (u + e) P^T |dO|,   |dQ~ - dQ| <= E |K|,   |dK~ - dK| <= E^T |Q|

(|X| elementwise, products of absolute matrices; dK and dV of a key/value head
sum over its query heads), plus 1e-6 absolute.  This module holds test
arithmetic only; the expected gradients come from the backward oracle.
"""
from __future__ import annotations

import numpy as np

U_BF16 = 2.0 ** -8
EPS = 2e-5


def bounds(q, k, v, dout, causal: bool, scale: float, k_len=None, row_chunk: int = 4096):
    """(bound_dq [B,H,N,d], bound_dk, bound_dv [B,H_kv,Nk,d]) for float64 arrays
    q, dout [B,H,N,d] and k, v [B,H_kv,Nk,d]; scale is the float32 softmax scale.

    Query rows are taken `row_chunk` at a time (every quantity of a row depends
    on that row alone; the dK and dV bounds add the chunks' contributions), so
    long sequences need O(row_chunk * Nk) memory instead of O(N * Nk)."""
    B, H, N, d = q.shape
    H_kv, Nk = k.shape[1], k.shape[2]
    g = H // H_kv
    bq = np.zeros_like(q)
    bk = np.zeros_like(k)
    bv = np.zeros_like(v)
    for b in range(B):
        L = Nk if k_len is None else min(max(int(k_len[b]), 0), Nk)
        for h in range(H):
            hk = h // g
            for r0 in range(0, N, row_chunk):
                r1 = min(N, r0 + row_chunk)
                allowed = np.zeros((r1 - r0, Nk), dtype=bool)
                allowed[:, :L] = True
                if causal:
                    allowed &= np.arange(Nk)[None, :] <= (np.arange(r0, r1)[:, None] + Nk - N)
                s = scale * q[b, h, r0:r1] @ k[b, hk].T
                s = np.where(allowed, s, -np.inf)
                m = s.max(axis=1, keepdims=True)
                live = np.isfinite(m[:, 0])
                e = np.where(allowed, np.exp(s - np.where(live[:, None], m, 0.0)), 0.0)
                P = e / np.where(live[:, None], e.sum(axis=1, keepdims=True), 1.0)
                O = P @ v[b, hk]
                dP = dout[b, h, r0:r1] @ v[b, hk].T
                D = (dout[b, h, r0:r1] * O).sum(axis=1, keepdims=True)
                dS = scale * P * (dP - D)
                absdo = np.abs(dout[b, h, r0:r1])
                A = absdo @ np.abs(v[b, hk]).T + (absdo * np.abs(O)).sum(axis=1, keepdims=True)
                E = (2 * U_BF16 + EPS) * np.abs(dS) + scale * P * EPS * A
                bq[b, h, r0:r1] = E @ np.abs(k[b, hk]) + 1e-6
                bk[b, hk] += E.T @ np.abs(q[b, h, r0:r1])
                bv[b, hk] += (U_BF16 + EPS) * (P.T @ absdo)
    return bq, bk + 1e-6, bv + 1e-6
