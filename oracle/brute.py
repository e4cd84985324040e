"""Scalar-loop restatement of the fast-weight MLP forward, for tiny shapes.

TEST INFRASTRUCTURE ONLY (see ``oracle/ittt_oracle.py``).  It uses no numpy
arithmetic: Python floats and explicit loops over tokens, channels and
hidden units, following the same pages and readings as the numpy oracle
([notes] gated-MLP, update and target equations; [review] sections 3-4;
[forum] item 3).  Intended for T <= 32, d <= 8, f <= 16.
"""

from __future__ import annotations

import math
from typing import List, Tuple


def _silu(x: float) -> float:
    if x >= 0:
        return x / (1.0 + math.exp(-x))
    e = math.exp(x)
    return x * e / (1.0 + e)


def forward_one(H, X0, W_gate, W_up, W_down0, conv, W_target, eta: float, C: int,
                clip: float = 0.0, chunk_pad: bool = False
                ) -> Tuple[List[List[float]], List[List[float]]]:
    """One sequence; all arguments are nested lists (or arrays indexable as [i][j]).

    chunk_pad: the conv's look-ahead stops at the end of each chunk."""
    T = len(H)
    d = len(H[0])
    f = len(W_gate)
    k = len(conv[0])
    W = [[float(W_down0[a][j]) for j in range(f)] for a in range(d)]
    O = [[0.0] * d for _ in range(T)]

    def z_row(t):
        z = []
        for j in range(f):
            g = 0.0
            u = 0.0
            for c in range(d):
                g += float(H[t][c]) * float(W_gate[j][c])
                u += float(H[t][c]) * float(W_up[j][c])
            z.append(_silu(g) * u)
        return z

    def v_row(t):
        limit = min(T, (t // C + 1) * C) if chunk_pad else T
        y = []
        for c in range(d):
            acc = 0.0
            for j in range(k):
                if t + j < limit:
                    acc += float(conv[c][j]) * float(X0[t + j][c])
            y.append(acc)
        v = []
        for o in range(d):
            acc = 0.0
            for c in range(d):
                acc += y[c] * float(W_target[c][o])
            v.append(acc)
        return v

    start = 0
    while start < T:
        end = min(start + C, T)
        zs = {t: z_row(t) for t in range(start, end)}
        # apply: every token of the chunk sees the state before the chunk's update
        for t in range(start, end):
            for a in range(d):
                acc = 0.0
                for j in range(f):
                    acc += zs[t][j] * W[a][j]
                O[t][a] = acc
        # update: W[a][j] += eta * sum_t Vhat[t][a] * Z[t][j], the delta's
        # Frobenius norm bounded by clip when clip > 0
        delta = [[0.0] * f for _ in range(d)]
        for t in range(start, end):
            v = v_row(t)
            for a in range(d):
                for j in range(f):
                    delta[a][j] += eta * v[a] * zs[t][j]
        scale = 1.0
        if clip > 0:
            nrm = math.sqrt(sum(x * x for row in delta for x in row))
            if nrm > clip:
                scale = clip / nrm
        for a in range(d):
            for j in range(f):
                W[a][j] += scale * delta[a][j]
        start = end
    return O, W
