"""Pure-Python brute force of the Avey-B ranker and layer, for tiny inputs.

Written independently of ``oracle/avey_oracle.c`` (plain lists, ``math`` only,
no shared helper) so that the two can pin each other.  Definitions follow the
Avey-B pages: MaxSim over split pairs (paperlayer summary §3; papernotes
整体框架), top-k with divide-by-max weights, eq. 8 compression with residual
(papernotes 关键设计 4), enricher ReLU^2, static V Z_t / dynamic eq. 6 mix,
fuser [Z_h || c] O + residual (papernotes 整体框架, 关键设计 2-3).
"""
import math


def _unit(v):
    n = math.sqrt(sum(a * a for a in v))
    n = max(n, 1e-12)
    return [a / n for a in v]


def _row(X, b, N, S, c, j, d):
    tok = c * S + j
    return list(X[b][tok]) if tok < N else [0.0] * d


def maxsim_matrix(X, S):
    """scores[b][t][c] by the definition (pad rows are zero vectors)."""
    B, N, d = len(X), len(X[0]), len(X[0][0])
    n = -(-N // S)
    out = []
    for b in range(B):
        rows = [[_unit(_row(X, b, N, S, c, j, d)) for j in range(S)] for c in range(n)]
        sc = []
        for t in range(n):
            line = []
            for c in range(n):
                tot = 0.0
                for i in range(S):
                    best = max(sum(p * q for p, q in zip(rows[t][i], rows[c][j])) for j in range(S))
                    tot += best
                line.append(tot)
            sc.append(line)
        out.append(sc)
    return out


def topk(scores_row, t, k, causal=False):
    cands = sorted(((-s, c) for c, s in enumerate(scores_row) if c != t and (not causal or c < t)))
    picked = cands[:k]
    s1 = -picked[0][0] if picked else 1.0
    s1 = s1 if s1 > 1e-30 else 1e-30
    idx = [c for _, c in picked] + [-1] * (k - len(picked))
    w = [(-ns) / s1 for ns, _ in picked] + [0.0] * (k - len(picked))
    return idx, w


def compress(X, S, k, b, t, idx, w, P):
    N, d = len(X[0]), len(X[0][0])
    blocks = [_row(X, b, N, S, t, j, d) for j in range(S)]
    for r in range(k):
        c = idx[r]
        for j in range(S):
            blocks.append([w[r] * a for a in _row(X, b, N, S, c, j, d)] if c >= 0 else [0.0] * d)
    out = []
    for i in range(S):
        acc = list(blocks[i])  # residual X_t
        for jj in range(len(blocks)):
            coef = P[i][jj]
            acc = [a + coef * v for a, v in zip(acc, blocks[jj])]
        out.append(acc)
    return out


def layer(x, U, bU, V, O, m_h, kind, eps, prenorm):
    S, d, m = len(x), len(x[0]), len(bU)
    xin = []
    for r in x:
        sc = 1.0 / math.sqrt(sum(a * a for a in r) / d + 1e-6) if prenorm else 1.0
        xin.append([a * sc for a in r])
    Z = []
    for r in xin:
        zr = []
        for f in range(m):
            a = bU[f] + sum(r[q] * U[q][f] for q in range(d))
            zr.append(max(a, 0.0) ** 2)
        Z.append(zr)
    Zh = [r[:m_h] for r in Z]
    Zt = [r[m_h:] for r in Z]
    mt = m - m_h
    if kind == 0:
        c = [[sum(V[i][j] * Zt[j][f] for j in range(S)) for f in range(mt)] for i in range(S)]
    elif kind == 2:  # coupled causal (original Avey)
        u = [_unit(r) for r in Zt]
        M = [[V[i][j] * sum(p * q for p, q in zip(u[i], u[j])) if j <= i else 0.0
              for j in range(S)] for i in range(S)]
        c = [[sum(M[i][j] * Zt[j][f] for j in range(S)) for f in range(mt)] for i in range(S)]
    else:
        u = [_unit(r) for r in Zt]
        G = [[sum(p * q for p, q in zip(u[i], u[j])) for j in range(S)] for i in range(S)]
        Gt = [[g / (sum(G[i]) + eps) for g in G[i]] for i in range(S)]
        c = [[sum(Gt[i][j] * Zt[j][f] for j in range(S)) for f in range(mt)] for i in range(S)]
    out = []
    for i in range(S):
        cat = Zh[i] + c[i]
        out.append([x[i][q] + sum(cat[f] * O[f][q] for f in range(m)) for q in range(d)])
    return out


def context(X, S, k, b, t, idx, w):
    """[X_t ; w_1 X_c1 ; ... ; w_k X_ck] as a list of (k+1)S rows."""
    N, d = len(X[0]), len(X[0][0])
    rows = [_row(X, b, N, S, t, j, d) for j in range(S)]
    for r in range(k):
        c = idx[r]
        for j in range(S):
            rows.append([w[r] * a for a in _row(X, b, N, S, c, j, d)] if c >= 0 else [0.0] * d)
    return rows
