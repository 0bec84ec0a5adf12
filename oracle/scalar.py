"""Literal scalar loops for tiny shapes (oracle; test infrastructure only).

These restate the same definitions as ``ssm``, ``mask`` and ``attention`` one
number at a time, with no numpy vectorisation, so that the vectorised oracle
can be brute-force checked on tiny inputs.  Sources and readings are those of
the modules they mirror (pith.science review of Attamba, "What carries the
argument", "Core claim"; Mamba's selective SSM named in "Assumptions & free
parameters").
"""

import math


def softplus(z):
    return z if z > 20.0 else math.log1p(math.exp(z))


def scan(u, dt, bias, A, Bm, Cm, starts):
    """u, dt: T x D nested lists; A: D x N; Bm, Cm: T x N; starts: set of chunk-start indices."""
    T, D, N = len(u), len(u[0]), len(A[0])
    h = [[0.0] * N for _ in range(D)]
    y = [[0.0] * D for _ in range(T)]
    for t in range(T):
        if t in starts:
            h = [[0.0] * N for _ in range(D)]
        for d in range(D):
            delta = softplus(dt[t][d] + bias[d])
            acc = 0.0
            for n in range(N):
                h[d][n] = math.exp(delta * A[d][n]) * h[d][n] + delta * u[t][d] * Bm[t][n]
                acc += Cm[t][n] * h[d][n]
            y[t][d] = acc
    return y


def in_mask(i, j, starts, n, L, mode):
    """One entry of M_train / M_test, from the definition."""
    if j > i:
        return False
    st = sorted(starts)
    def chunk(p):
        c = 0
        for k, s in enumerate(st):
            if s <= p:
                c = k
        return c
    ends = [s - 1 for s in st[1:]] + [n - 1]
    is_boundary = j == ends[chunk(j)]
    in_window = (i - j) < L
    if mode == "train":
        return is_boundary or chunk(j) == chunk(i) or in_window
    return is_boundary or in_window


def attention(q, k, v, allowed, scale):
    """q, k, v: n x dh nested lists (one head); allowed(i, j) -> bool.  Returns O (n x dh)."""
    n, dh = len(q), len(q[0])
    out = []
    for i in range(n):
        keys = [j for j in range(n) if allowed(i, j)]
        if not keys:
            out.append([0.0] * dh)
            continue
        s = [sum(q[i][c] * k[j][c] for c in range(dh)) * scale for j in keys]
        m = max(s)
        w = [math.exp(x - m) for x in s]
        z = sum(w)
        out.append([sum(w[a] * v[keys[a]][c] for a in range(len(keys))) / z for c in range(dh)])
    return out


def project(x, W):
    """y[m, o] = sum_k x[m, k] W[o, k], one number at a time (brute force for tiny shapes)."""
    M, K = len(x), len(x[0])
    out = [[0.0] * len(W) for _ in range(M)]
    for m in range(M):
        for o in range(len(W)):
            acc = 0.0
            for k in range(K):
                acc += float(x[m][k]) * float(W[o][k])
            out[m][o] = acc
    return out
