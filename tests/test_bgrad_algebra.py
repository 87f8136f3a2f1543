"""The chunk-form backward's algebra, step by step, against the chunkwise
fp64 adjoint (oracle/chunkwise_adjoint.py, itself pinned to the token sweep).

The per-chunk gradient kernel evaluates the chunk's gradients through a chain
of dense products and reformulations: Delta = u0 - w S0^T, U from Delta and
the Gram, Dd = T^T (diag(dn) K Y^T) + N1 dO with N1 = T^T M, the X1 / X23 / Xq
coefficient matrices, and dalpha through F = (E1 - E2b) D + E2b and the psi
expansion; the last chunk of a sequence is padded with k = q = v = dO = 0,
alpha = 1, beta = 0.  This test writes those steps out in fp64 numpy
(0-indexed tokens, as the kernel indexes them) and checks them against
chunk_backward on whole and padded chunks, with a reset token (alpha = 0)
and a write token (beta = 1), to rounding.  A dropped term, a transposed
coefficient matrix or a wrong decay index in the reformulation fails it.
"""
import numpy as np
import pytest

from oracle.chunkwise_adjoint import chunk_backward


def chunk_form(S0, Y, q, k, v, a, b, dO, C):
    n = k.shape[0]

    def pad(x, val=0.0):
        return np.concatenate([x, np.full((C - n,) + x.shape[1:], val)]) if n < C else x

    q, k, v, dO = pad(q), pad(k), pad(v), pad(dO)
    a, b = pad(a, 1.0), pad(b, 0.0)
    DM = np.zeros((C, C))                       # D[t][s] = a_{s+1} ... a_t
    for s in range(C):
        DM[s, s] = 1.0
        for t in range(s + 1, C):
            DM[t, s] = DM[t - 1, s] * a[t]
    g = np.array([np.prod(a[:t + 1]) for t in range(C)])
    gp = np.concatenate([[1.0], g[:-1]])
    dn = np.array([np.prod(a[t + 1:]) for t in range(C)])
    KK, KQ = k @ k.T, k @ q.T
    T = np.linalg.inv(np.eye(C) + np.tril(b[:, None] * DM * KK, -1))
    u0, w = T @ (b[:, None] * v), T @ ((b * g)[:, None] * k)
    E, KS, KY = S0 @ w.T, S0 @ k.T, Y @ k.T       # [i][t]
    Delta = u0 - E.T
    cv = np.sum(Delta * KY.T, axis=1)
    N1 = T.T @ np.triu(DM.T * KQ)                 # M[s][u] = D[u][s] KQ[s][u], u >= s
    Xu = np.zeros((C, C))
    for t in range(1, C):
        Xu[t, :t] = DM[t - 1, :t] * KK[:t, t]
    UT = gp[None, :] * KS + Delta.T @ Xu.T
    DdT = np.concatenate([dn[None, :] * KY, dO.T], axis=1) @ np.concatenate([T.T, N1], axis=1).T
    Dd = DdT.T
    dv = b[:, None] * Dd
    dbeta = np.sum(Dd * (v - a[:, None] * UT.T), axis=1)
    du, bv = np.sum(Dd * UT.T, axis=1), np.sum(Dd * KS.T, axis=1)
    q1 = S0.T @ dO.T
    av = np.sum(q1.T * q, axis=1)
    dqT = g[None, :] * q1
    dkT = S0.T @ ((-(a * b) * gp)[:, None] * Dd).T + Y.T @ (dn[:, None] * Delta).T
    DOD, DDD = dO @ Delta.T, Dd @ Delta.T
    X1, X23, Xq = np.zeros((C, C)), np.zeros((C, C)), np.zeros((C, C))
    for t in range(C):
        for s in range(C):
            if s >= t:
                X1[t, s] = DM[s, t] * DOD[s, t]
            if s > t:
                X23[t, s] = DM[s, t] * b[s] * DDD[s, t]
            if s < t:
                X23[t, s] = a[t] * b[t] * DM[t - 1, s] * DDD[t, s]
            if s <= t:
                Xq[t, s] = DM[t, s] * DOD[t, s]
    dkT += np.concatenate([q.T, k.T], axis=1) @ np.concatenate([X1, -X23], axis=1).T
    dqT += k.T @ Xq.T
    E2b = b[None, :] * DDD.T * KK                 # E2b[r][s] = beta_s (Delta_r . Dd_s)(k_r . k_s)
    F = (DOD.T * KQ - E2b) @ DM + E2b             # (E1 - E2b) D + E2b
    YS = np.sum(Y * S0)
    dalpha = np.zeros(C)
    for t in range(C):
        acc = dn[t] * YS + sum(DM[s, t] * (av[s] - b[s] * bv[s]) for s in range(t, C)) + b[t] * bv[t]
        psi = gp[t] * acc + sum(DM[t - 1, r] * (dn[t] * cv[r] + F[r, t]) for r in range(t))
        dalpha[t] = psi - b[t] * du[t]
    return dqT.T[:n], dkT.T[:n], dv[:n], dalpha[:n], dbeta[:n]


@pytest.mark.parametrize("d,C,n", [(8, 16, 16), (8, 16, 11), (16, 32, 32), (16, 32, 5), (4, 16, 1)])
def test_chunk_form_steps_match_the_chunkwise_adjoint(d, C, n):
    rng = np.random.default_rng(100 * d + n)
    S0, Y = rng.standard_normal((d, d)), rng.standard_normal((d, d))
    q, k, v, dO = (rng.standard_normal((n, d)) / np.sqrt(d) for _ in range(4))
    a, b = rng.uniform(0.3, 1.0, n), rng.uniform(0.0, 1.0, n)
    a[n // 2] = 0.0          # a reset
    b[(n - 1) // 3] = 1.0    # a write
    ref = chunk_backward(S0, Y, q, k, v, a, b, dO)
    got = chunk_form(S0, Y, q, k, v, a, b, dO, C)
    for name, r, x in zip(("dq", "dk", "dv", "dalpha", "dbeta"), ref[:5], got):
        assert np.max(np.abs(r - x)) <= 1e-12 * max(np.max(np.abs(r)), 1.0), name
