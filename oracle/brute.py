"""Pure-Python loop spelling of the attention definition (test infrastructure).

For tiny shapes only (n <= ~16, d <= ~8).  Written with scalar loops and the
math module, independently of the vectorised code in ``attention.py``, so the
two can check each other: a transposed operand or a dropped term in one of
them shows up as a mismatch.  Formulas: sigmoid attention and its bias,
"Better Models, Faster Training", sections 2A-2B; softmax and softmax_1, the
QuietAttention page, section "Proposition : softmax_1 et QuietAttention".
"""
from __future__ import annotations

import math

SIGMOID, SOFTMAX, SOFTMAX1 = 0, 1, 2


def _sig(x):
    if x >= 0:
        return 1.0 / (1.0 + math.exp(-x))
    e = math.exp(x)
    return e / (1.0 + e)


def _weights_row(srow, mrow, epilogue):
    n = len(srow)
    keys = [j for j in range(n) if mrow[j]]
    p = [0.0] * n
    if not keys:
        return p
    if epilogue == SIGMOID:
        for j in keys:
            p[j] = _sig(srow[j])
        return p
    mx = max(srow[j] for j in keys)
    if epilogue == SOFTMAX1:
        mx = max(mx, 0.0)
    den = sum(math.exp(srow[j] - mx) for j in keys)
    if epilogue == SOFTMAX1:
        den += math.exp(0.0 - mx)
    for j in keys:
        p[j] = math.exp(srow[j] - mx) / den
    return p


def forward_head(q, k, v, mask, bias, scale, epilogue):
    """Lists of lists: q [Nq][d], k [Nk][d], v [Nk][dv], mask [Nq][Nk], bias [Nq]."""
    Nq, Nk, dv = len(q), len(k), len(v[0])
    P = []
    O = []
    for i in range(Nq):
        srow = [scale * sum(q[i][t] * k[j][t] for t in range(len(q[i]))) + bias[i]
                for j in range(Nk)]
        p = _weights_row(srow, mask[i], epilogue)
        P.append(p)
        O.append([sum(p[j] * v[j][c] for j in range(Nk)) for c in range(dv)])
    return O, P


def backward_head(q, k, v, do, mask, bias, scale, epilogue):
    Nq, Nk, d, dv = len(q), len(k), len(q[0]), len(v[0])
    O, P = forward_head(q, k, v, mask, bias, scale, epilogue)
    dQ = [[0.0] * d for _ in range(Nq)]
    dK = [[0.0] * d for _ in range(Nk)]
    dV = [[0.0] * dv for _ in range(Nk)]
    for i in range(Nq):
        Di = sum(do[i][c] * O[i][c] for c in range(dv))
        for j in range(Nk):
            p = P[i][j]
            if p == 0.0 and not mask[i][j]:
                continue
            dp = sum(do[i][c] * v[j][c] for c in range(dv))
            if epilogue == SIGMOID:
                ds = dp * p * (1.0 - p)
            else:
                ds = p * (dp - Di)
            for c in range(dv):
                dV[j][c] += p * do[i][c]
            for t in range(d):
                dQ[i][t] += scale * ds * k[j][t]
                dK[j][t] += scale * ds * q[i][t]
    return dQ, dK, dV
