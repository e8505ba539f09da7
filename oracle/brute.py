"""Pure-Python brute force for tiny inputs (N <= 8): a second, loop-level oracle.

Test infrastructure only (see the package docstring). No NumPy in the
arithmetic: nested lists and the math module, so it shares no vectorised code
path with taylor_la.py / swa.py. Used to pin them on tiny cases.
"""

from __future__ import annotations

import math


def phi(x):
    """[1, x_0..x_{d-1}, x_a*x_b/sqrt(2) for a in 0..d-1 for b in 0..d-1]."""
    out = [1.0]
    out.extend(float(t) for t in x)
    r = 1.0 / math.sqrt(2.0)
    for a in range(len(x)):
        for b in range(len(x)):
            out.append(float(x[a]) * float(x[b]) * r)
    return out


def dot(a, b):
    acc = 0.0
    for s, t in zip(a, b):
        acc += float(s) * float(t)
    return acc


def la(q, k, v):
    """One head: q, k lists of N vectors of length d', v list of N vectors.

    Builds phi explicitly for every token and evaluates
    y_i = sum_{j<=i} (phi(q_i).phi(k_j)) v_j / sum_{j<=i} phi(q_i).phi(k_j),
    plus S = sum_j phi(k_j) v_j^T and z = sum_j phi(k_j).
    Returns (y, S, z) as nested lists.
    """
    n = len(q)
    dv = len(v[0])
    fq = [phi(x) for x in q]
    fk = [phi(x) for x in k]
    y = []
    for i in range(n):
        num = [0.0] * dv
        den = 0.0
        for j in range(i + 1):
            a = dot(fq[i], fk[j])
            den += a
            for e in range(dv):
                num[e] += a * float(v[j][e])
        y.append([t / den for t in num])
    D = len(fk[0])
    S = [[0.0] * dv for _ in range(D)]
    z = [0.0] * D
    for j in range(n):
        for f in range(D):
            z[f] += fk[j][f]
            for e in range(dv):
                S[f][e] += fk[j][f] * float(v[j][e])
    return y, S, z


def swa(q, k, v, w, scale):
    """One head, window of w keys ending at the query: exact softmax with math.exp."""
    n = len(q)
    dv = len(v[0])
    y = []
    for i in range(n):
        js = [j for j in range(n) if i - w < j <= i]
        s = [scale * dot(q[i], k[j]) for j in js]
        m = max(s)
        e = [math.exp(t - m) for t in s]
        tot = sum(e)
        row = [0.0] * dv
        for p, j in zip(e, js):
            for c in range(dv):
                row[c] += p / tot * float(v[j][c])
        y.append(row)
    return y
