"""Pure-Python fp64 model of the tiled online-softmax recurrence.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Follows the page "FlashAttention (ES)": section "Tiling y procesamiento por
bloques" (keys are visited block by block, the result is updated after each
block, the score matrix is never stored whole) and section "Calculo de Softmax
en linea" (two running values -- the current maximum and the sum of
exponentials -- are updated as each block arrives, and the final result is the
exact softmax).  The pages state the idea without formulas; the update written
here is the plainest reading that keeps the result exact: when the running
maximum moves from m to m', everything accumulated so far is multiplied by
exp(m - m') before the new block's terms, taken relative to m', are added.

Scalar Python loops: for tiny inputs only (the brute-force pin).
"""
from __future__ import annotations

import math


def attention_online(q, k, v, causal: bool, scale: float, k_len=None, tile: int = 1):
    """Online-softmax attention over key blocks of ``tile`` keys.

    q, k, v: nested sequences (or arrays) of floats shaped [B][H][N][d].
    Returns (O [B][H][N][d], lse [B][H][N]) as nested lists of Python floats.
    Rows with no allowed key give O = 0 and lse = -inf.
    """
    if tile < 1:
        raise ValueError("tile must be >= 1")
    B, H, N, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    sigma = float(scale)
    O = [[[[0.0] * d for _ in range(N)] for _ in range(H)] for _ in range(B)]
    LSE = [[[-math.inf] * N for _ in range(H)] for _ in range(B)]
    for b in range(B):
        L = N if k_len is None else max(0, min(N, int(k_len[b])))
        for h in range(H):
            for i in range(N):
                m = -math.inf          # running maximum
                l = 0.0                # running sum of exp(s - m)
                acc = [0.0] * d        # running sum of exp(s - m) * v
                for start in range(0, N, tile):
                    # scores of this block; masked keys are -inf
                    blk = []
                    for j in range(start, min(start + tile, N)):
                        if j >= L or (causal and j > i):
                            blk.append((j, -math.inf))
                        else:
                            s = sigma * sum(float(q[b][h][i][t]) * float(k[b][h][j][t]) for t in range(d))
                            blk.append((j, s))
                    m_blk = max(s for _, s in blk)
                    if m_blk == -math.inf:
                        continue       # a fully masked block contributes exactly 0
                    m_new = max(m, m_blk)
                    alpha = 0.0 if m == -math.inf else math.exp(m - m_new)
                    l *= alpha
                    acc = [a * alpha for a in acc]
                    for j, s in blk:
                        if s == -math.inf:
                            continue
                        p = math.exp(s - m_new)
                        l += p
                        for t in range(d):
                            acc[t] += p * float(v[b][h][j][t])
                    m = m_new
                if l > 0.0:
                    O[b][h][i] = [a / l for a in acc]
                    LSE[b][h][i] = m + math.log(l)
    return O, LSE
