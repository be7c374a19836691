"""Scalar triple-loop attention in pure Python, for tiny inputs.

TEST INFRASTRUCTURE ONLY (see ``oracle/attention.py``).  This is the
attention definition written element by element with ``math.exp`` and
Python floats (IEEE double) and no numpy.  Each row first gets its
log-sum-exp in a separate pass, then P_ij = exp(s_ij - lse_i); the backward
is derived directly from the scalar chain rule:

  O_ic   = sum_j P_ij V_jc,            P_ij = exp(s_ij - lse_i)
  s_ij   = scale sum_c Q_ic K_jc       (j <= i only when causal)
  dV_jc  = sum_i P_ij dO_ic
  dP_ij  = sum_c dO_ic V_jc
  dS_ij  = P_ij (dP_ij - sum_t P_it dP_it)
  dQ_ic  = scale sum_j dS_ij K_jc,     dK_jc = scale sum_i dS_ij Q_ic

It is only used to pin the vectorised oracle at N <= 16.
"""
from __future__ import annotations

import math
from typing import List, Tuple

Mat = List[List[float]]


def _to_lists(x) -> Mat:
    if hasattr(x, "tolist"):
        if hasattr(x, "detach"):
            x = x.detach().cpu().double()
        return [[float(e) for e in row] for row in x.tolist()]
    return [[float(e) for e in row] for row in x]


def _visible(i: int, j: int, causal: bool) -> bool:
    return (not causal) or j <= i


def forward(q, k, v, scale: float, causal: bool) -> Tuple[Mat, List[float]]:
    q, k, v = _to_lists(q), _to_lists(k), _to_lists(v)
    n, nk, dv = len(q), len(k), len(v[0])
    o: Mat = []
    lse: List[float] = []
    for i in range(n):
        s = {}
        for j in range(nk):
            if _visible(i, j, causal):
                acc = 0.0
                for c in range(len(q[i])):
                    acc += q[i][c] * k[j][c]
                s[j] = scale * acc
        top = max(s.values())
        total = 0.0
        for j in s:
            total += math.exp(s[j] - top)
        z = top + math.log(total)
        lse.append(z)
        row = [0.0] * dv
        for j in s:
            w = math.exp(s[j] - z)
            for c in range(dv):
                row[c] += w * v[j][c]
        o.append(row)
    return o, lse


def backward(q, k, v, do, scale: float, causal: bool) -> Tuple[Mat, Mat, Mat]:
    q, k, v, do = _to_lists(q), _to_lists(k), _to_lists(v), _to_lists(do)
    n, nk, d, dvd = len(q), len(k), len(q[0]), len(v[0])
    _, lse = forward(q, k, v, scale, causal)
    dq = [[0.0] * d for _ in range(n)]
    dk = [[0.0] * d for _ in range(nk)]
    dv = [[0.0] * dvd for _ in range(nk)]
    for i in range(n):
        p = {}
        for j in range(nk):
            if _visible(i, j, causal):
                acc = 0.0
                for c in range(d):
                    acc += q[i][c] * k[j][c]
                p[j] = math.exp(scale * acc - lse[i])
        dp = {}
        for j in p:
            acc = 0.0
            for c in range(dvd):
                acc += do[i][c] * v[j][c]
            dp[j] = acc
        inner = 0.0
        for j in p:
            inner += p[j] * dp[j]
        for j in p:
            ds = p[j] * (dp[j] - inner)
            for c in range(dvd):
                dv[j][c] += p[j] * do[i][c]
            for c in range(d):
                dq[i][c] += scale * ds * k[j][c]
                dk[j][c] += scale * ds * q[i][c]
    return dq, dk, dv
