"""Pure-Python brute-force attention for tiny shapes (test infrastructure only).

Scalar loops over every (i, j, c) index, written straight from the definition
softmax(Q K^T * scale) V ("FlashAttention — フラッシュアテンション", section
標準的なアテンションの問題点) and from the chain rule of L = sum(O * dO).  It
uses no array library at all, so it shares nothing with the NumPy oracle it is
compared against.  Intended for N <= 16, d <= 8.
"""
from __future__ import annotations

import math


def _visible(i: int, j: int, causal: bool) -> bool:
    return (not causal) or j <= i


def brute_fwd(q, k, v, scale: float, causal: bool):
    """q, k, v: nested lists [N][d] of floats for ONE head.  Returns (O [N][dv], LSE [N])."""
    N, Nk, dv = len(q), len(k), len(v[0])
    O, LSE = [], []
    for i in range(N):
        s = []
        for j in range(Nk):
            if _visible(i, j, causal):
                acc = 0.0
                for c in range(len(q[i])):
                    acc += q[i][c] * k[j][c]
                s.append(acc * scale)
            else:
                s.append(None)
        m = max(x for x in s if x is not None)
        e = [0.0 if x is None else math.exp(x - m) for x in s]
        den = sum(e)
        O.append([sum(e[j] / den * v[j][c] for j in range(Nk)) for c in range(dv)])
        LSE.append(m + math.log(den))
    return O, LSE


def brute_bwd(q, k, v, do, scale: float, causal: bool):
    """Gradients of L = sum_ic O_ic dO_ic for ONE head, by explicit index sums."""
    N, Nk, d, dv = len(q), len(k), len(q[0]), len(v[0])
    P = []
    for i in range(N):
        s = [sum(q[i][c] * k[j][c] for c in range(d)) * scale if _visible(i, j, causal) else None
             for j in range(Nk)]
        m = max(x for x in s if x is not None)
        e = [0.0 if x is None else math.exp(x - m) for x in s]
        den = sum(e)
        P.append([x / den for x in e])
    dV = [[sum(P[i][j] * do[i][c] for i in range(N)) for c in range(dv)] for j in range(Nk)]
    dP = [[sum(do[i][c] * v[j][c] for c in range(dv)) for j in range(Nk)] for i in range(N)]
    D = [sum(P[i][j] * dP[i][j] for j in range(Nk)) for i in range(N)]
    dS = [[P[i][j] * (dP[i][j] - D[i]) for j in range(Nk)] for i in range(N)]
    dQ = [[scale * sum(dS[i][j] * k[j][c] for j in range(Nk)) for c in range(d)] for i in range(N)]
    dK = [[scale * sum(dS[i][j] * q[i][c] for i in range(N)) for c in range(d)] for j in range(Nk)]
    return dQ, dK, dV


def brute_decode(q, k, v, scale: float, causal: bool):
    """One query head against its key/value head, queries at the END of the sequence.

    q: [Nq][d], k, v: [Nk][d] nested lists.  Query i sits at position Nk - Nq + i, so
    with causal it sees keys j <= Nk - Nq + i.  Returns (O [Nq][dv], LSE [Nq]).
    """
    Nq, Nk, dv = len(q), len(k), len(v[0])
    O, LSE = [], []
    for i in range(Nq):
        pos = Nk - Nq + i
        s = []
        for j in range(Nk):
            if causal and j > pos:
                s.append(None)
                continue
            acc = 0.0
            for c in range(len(q[i])):
                acc += q[i][c] * k[j][c]
            s.append(acc * scale)
        m = max(x for x in s if x is not None)
        e = [0.0 if x is None else math.exp(x - m) for x in s]
        den = sum(e)
        O.append([sum(e[j] / den * v[j][c] for j in range(Nk)) for c in range(dv)])
        LSE.append(m + math.log(den))
    return O, LSE
