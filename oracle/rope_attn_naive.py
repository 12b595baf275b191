"""Explicit-loop float64 oracle for tiny problems (n <= 32, one head at a time).

TEST INFRASTRUCTURE ONLY (see ``oracle/rope_attn_ref.py`` for the rule and
the definitions).  It restates the same definitions scalar by scalar, with no
numpy linear algebra, so that an indexing or blocking slip in the vectorised
oracle shows up as a disagreement.  The pairing of coordinates into bands is
the interleaved one, (2m, 2m+1).

Sources: "RoPE attention can be trained in almost-linear time" (Metodologia 1:
normalised softmax s(x), error term l(x), beta(x), gamma(x) = diag(s) beta -
s s^T beta); "LeRoPE: learnable RoPE frequencies" (Mecanismo Central:
theta_hat_m = exp(alpha_m) theta_m; Escolhas de Design Principais: d/2
frequencies shared by all heads).
"""
import math


def _rot(x0, x1, a):
    c, s = math.cos(a), math.sin(a)
    return c * x0 - s * x1, s * x0 + c * x1


def head(q, k, v, e, alpha, base, causal):
    """One head: q, k, v, e are n x d nested lists.  Returns a dict of results."""
    n, d = len(q), len(q[0])
    M = d // 2
    th = [math.exp(alpha[m]) * base ** (-2.0 * m / d) for m in range(M)]

    def rot_rows(x, sign):
        out = []
        for p in range(n):
            row = [0.0] * d
            for m in range(M):
                row[2 * m], row[2 * m + 1] = _rot(x[p][2 * m], x[p][2 * m + 1], sign * p * th[m])
            out.append(row)
        return out

    qt, kt = rot_rows(q, 1.0), rot_rows(k, 1.0)
    sc = 1.0 / math.sqrt(d)
    allowed = [[(not causal) or j <= i for j in range(n)] for i in range(n)]
    S = [[sum(qt[i][c] * kt[j][c] for c in range(d)) * sc for j in range(n)] for i in range(n)]
    P = []
    lse = []
    for i in range(n):
        ex = [math.exp(S[i][j]) if allowed[i][j] else 0.0 for j in range(n)]
        z = sum(ex)
        P.append([x / z for x in ex])
        lse.append(math.log(z))
    O = [[sum(P[i][j] * v[j][c] for j in range(n)) for c in range(d)] for i in range(n)]
    dO = [[O[i][c] - e[i][c] for c in range(d)] for i in range(n)]
    L = 0.5 * sum(dO[i][c] ** 2 for i in range(n) for c in range(d))
    beta = [[sum(dO[i][c] * v[j][c] for c in range(d)) for j in range(n)] for i in range(n)]
    dS = []
    for i in range(n):
        sb = sum(P[i][j] * beta[i][j] for j in range(n))
        dS.append([P[i][j] * beta[i][j] - P[i][j] * sb for j in range(n)])
    dV = [[sum(P[i][j] * dO[i][c] for i in range(n)) for c in range(d)] for j in range(n)]
    dQt = [[sum(dS[i][j] * kt[j][c] for j in range(n)) * sc for c in range(d)] for i in range(n)]
    dKt = [[sum(dS[i][j] * qt[i][c] for i in range(n)) * sc for c in range(d)] for j in range(n)]
    dQ, dK = rot_rows(dQt, -1.0), rot_rows(dKt, -1.0)
    dalpha = []
    for m in range(M):
        acc = 0.0
        for p in range(n):
            acc += p * (dQt[p][2 * m + 1] * qt[p][2 * m] - dQt[p][2 * m] * qt[p][2 * m + 1])
            acc += p * (dKt[p][2 * m + 1] * kt[p][2 * m] - dKt[p][2 * m] * kt[p][2 * m + 1])
        dalpha.append(th[m] * acc)
    return dict(o=O, lse=lse, L=L, do=dO, dq=dQ, dk=dK, dv=dV, dalpha=dalpha, P=P, dS=dS,
                S=S, qt=qt, kt=kt)
