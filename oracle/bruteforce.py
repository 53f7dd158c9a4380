"""Pure-Python nested-loop restatement of the LLA steps, for tiny inputs.

TEST INFRASTRUCTURE ONLY (see ``oracle/lla_oracle.py``).  No NumPy
arithmetic is used here: lists of Python floats and explicit loops, so that
the vectorised oracle can be checked against a second, independent
transcription of the same equations of "Looped Latent Attention: Cross-Loop
KV Compression for Looped Transformers" (arXiv 2607.15456).

The codec fit is restated as a cyclic Jacobi eigen-decomposition of the
centred calibration covariance: its leading eigenvectors span the same
subspace as the top right singular vectors the paper's SVD initialisation
takes [LLA §3, "Initialisation and conversion"].
"""

from __future__ import annotations

import math


def mean_rows(X):
    n = len(X)
    S = len(X[0])
    return [sum(X[i][k] for i in range(n)) / n for k in range(S)]


def jacobi_eigh(A, sweeps=100, tol=1e-15):
    """Eigen-decomposition of a small symmetric matrix by cyclic Jacobi rotations.

    Returns (eigenvalues, eigenvectors as columns), sorted by decreasing eigenvalue.
    """
    n = len(A)
    a = [row[:] for row in A]
    v = [[1.0 if i == j else 0.0 for j in range(n)] for i in range(n)]
    for _ in range(sweeps):
        off = sum(a[i][j] ** 2 for i in range(n) for j in range(n) if i != j)
        if off < tol:
            break
        for p in range(n - 1):
            for q in range(p + 1, n):
                if abs(a[p][q]) < 1e-300:
                    continue
                theta = (a[q][q] - a[p][p]) / (2.0 * a[p][q])
                t = (1.0 if theta >= 0 else -1.0) / (abs(theta) + math.sqrt(theta * theta + 1.0))
                c = 1.0 / math.sqrt(t * t + 1.0)
                s = t * c
                for k in range(n):
                    akp, akq = a[k][p], a[k][q]
                    a[k][p] = c * akp - s * akq
                    a[k][q] = s * akp + c * akq
                for k in range(n):
                    apk, aqk = a[p][k], a[q][k]
                    a[p][k] = c * apk - s * aqk
                    a[q][k] = s * apk + c * aqk
                for k in range(n):
                    vkp, vkq = v[k][p], v[k][q]
                    v[k][p] = c * vkp - s * vkq
                    v[k][q] = s * vkp + c * vkq
    vals = [a[i][i] for i in range(n)]
    order = sorted(range(n), key=lambda i: -vals[i])
    return [vals[i] for i in order], [[v[k][i] for i in order] for k in range(n)]


def fit_codec(X, r):
    """mu and a W_down [S][r] whose columns are the top-r principal directions."""
    mu = mean_rows(X)
    n, S = len(X), len(X[0])
    Xc = [[X[i][k] - mu[k] for k in range(S)] for i in range(n)]
    C = [[sum(Xc[i][a] * Xc[i][b] for i in range(n)) for b in range(S)] for a in range(S)]
    _, vecs = jacobi_eigh(C)
    W = [[vecs[k][a] for a in range(r)] for k in range(S)]
    return mu, W


def encode(x, mu, W):
    """c_a = sum_k (x_k - mu_k) W[k][a]   (eq. (2))."""
    S, r = len(W), len(W[0])
    return [sum((x[k] - mu[k]) * W[k][a] for k in range(S)) for a in range(r)]


def reconstruct(c, Wt, mut):
    """x_hat_i = sum_a c_a Wt[i][a] + mut_i   (eq. (3))."""
    return [sum(c[a] * Wt[i][a] for a in range(len(c))) + mut[i] for i in range(len(Wt))]


def rope(x, pos, base):
    d = len(x)
    h = d // 2
    y = [0.0] * d
    for i in range(h):
        th = pos * base ** (-2.0 * i / d)
        cs, sn = math.cos(th), math.sin(th)
        y[i] = x[i] * cs - x[i + h] * sn
        y[i + h] = x[i + h] * cs + x[i] * sn
    return y


def attention(q, Ks, Vs, scale):
    if not Ks:
        return [0.0] * (len(Vs[0]) if Vs else len(q))
    logits = [scale * sum(qi * ki for qi, ki in zip(q, k)) for k in Ks]
    m = max(logits)
    w = [math.exp(l - m) for l in logits]
    z = sum(w)
    dv = len(Vs[0])
    return [sum(w[j] * Vs[j][i] for j in range(len(Vs))) / z for i in range(dv)]


def decode_head(q, cK, cV, muKt, WKt, muVt, WVt, pos_q, scale, base, k_self=None, v_self=None):
    """Loop-t attention of one head over its cached latents (token j at position j), plus the
    current token's exact key and value as one more slot at the query's position when given."""
    Ks = [rope(reconstruct(c, WKt, muKt), j, base) for j, c in enumerate(cK)]
    Vs = [reconstruct(c, WVt, muVt) for c in cV]
    if k_self is not None:
        Ks.append(rope(list(k_self), pos_q, base))
        Vs.append(list(v_self))
    return attention(rope(q, pos_q, base), Ks, Vs, scale)
