"""A second, independent float64 statement of one mHC sublayer, in plain Python
loops, for tiny inputs only.  It is written straight from the mHC paper notes
(section 3 Eq.(3); section 4.2 Eq.(7)-(9)) and shares nothing with the oracle:
it uses Eq.(14)-(16)'s order (project raw x, then divide by r) where the
oracle normalises first, and keeps the Sinkhorn matrix as nested lists.
"""
from __future__ import annotations

import math


def _sinkhorn(logits, t_iters):
    n = len(logits)
    M = [[math.exp(v) for v in row] for row in logits]
    for _ in range(t_iters):
        col = [sum(M[i][j] for i in range(n)) for j in range(n)]
        M = [[M[i][j] / col[j] for j in range(n)] for i in range(n)]
        row = [sum(M[i]) for i in range(n)]
        M = [[M[i][j] / row[i] for j in range(n)] for i in range(n)]
    return M


def sublayer(Xt, Ft, phi, alpha, b, t_iters=20, eps=1e-6):
    """One token: Xt is n lists of C floats, Ft C floats, phi nC lists of P floats.
    Returns (x_in, H_pre, H_post, H_res, X_next)."""
    n, C = len(Xt), len(Xt[0])
    P = n * n + 2 * n
    flat = [Xt[i][c] for i in range(n) for c in range(C)]
    r = math.sqrt(sum(v * v for v in flat) / (n * C) + eps)
    proj = [sum(flat[q] * phi[q][p] for q in range(n * C)) for p in range(P)]
    z = []
    for p in range(P):
        a = alpha[0] if p < n else (alpha[1] if p < 2 * n else alpha[2])
        z.append(a * proj[p] / r + b[p])
    H_pre = [1.0 / (1.0 + math.exp(-z[i])) for i in range(n)]
    H_post = [2.0 / (1.0 + math.exp(-z[n + i])) for i in range(n)]
    H_res = _sinkhorn([[z[2 * n + i * n + j] for j in range(n)] for i in range(n)], t_iters)
    x_in = [sum(H_pre[i] * Xt[i][c] for i in range(n)) for c in range(C)]
    X_next = [[sum(H_res[i][j] * Xt[j][c] for j in range(n)) + H_post[i] * Ft[c]
               for c in range(C)] for i in range(n)]
    return x_in, H_pre, H_post, H_res, X_next
