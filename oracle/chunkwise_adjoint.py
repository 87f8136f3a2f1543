"""Chunkwise fp64 form of the gated delta rule's gradient -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's cpu_baseline leg may
import this module.

The second, independent form of the adjoint (the first is the token-by-token
reverse sweep in adjoint_fp64.c).  The loss is L = sum_t dO_t . o_t plus
<W, S_final> for a given final-state gradient W, through the recurrence of the
IsoExec summary page, section "Chunkwise-Parallel Recurrent (CPR) Gated
DeltaNet".  Everything is written per chunk as dense products of chunk-sized
matrices, the form a tensor-core backward evaluates, and it needs no division
and no logarithm of a gate (alpha = 0 is exact).

Inside a chunk of n tokens that starts from state S0 and ends with the
gradient Y for its end state, with decay products D[t, s] = alpha_{s+1} ...
alpha_t (D[t, t] = 1; token indices 1..n, 0 = the chunk start), derived here
from S_t = alpha_t S_{t-1} + delta_t k_t^T and G_{t-1} = alpha_t G_t -
alpha_t beta_t (G_t k_t) k_t^T + dO_{t-1} q_{t-1}^T:

* forward: (I + A) Delta = diag(beta) (V - diag(D[., 0]) K S0^T) with
  A[t, r] = beta_t D[t, r] (k_t . k_r) for r < t;  u_t = S_{t-1} k_t =
  D[t-1, 0] S0 k_t + sum_{r<t} D[t-1, r] (k_r . k_t) delta_r;
* backward: ddelta_t = H_t k_t, with H_t = dL/dS_t, solves
  (I + A^T) Ddelta = diag(D[n, .]) K Y^T + M Dout,
  M[t, s] = D[s, t] (k_t . q_s) for s >= t;
* dv = diag(beta) Ddelta;  dbeta_t = ddelta_t . (v_t - alpha_t u_t);
* dq_t = D[t, 0] S0^T dO_t + sum_{r<=t} D[t, r] (delta_r . dO_t) k_r;
* dk_t = D[n, t] Y^T delta_t + sum_{s>=t} D[s, t] (dO_s . delta_t) q_s
         - sum_{s>t} D[s, t] beta_s (ddelta_s . delta_t) k_s
         - alpha_t beta_t [D[t-1, 0] S0^T ddelta_t + sum_{r<t} D[t-1, r] (delta_r . ddelta_t) k_r];
* dalpha_t = <H_t, S_{t-1}> - beta_t ddelta_t . u_t, the inner product
  expanded into S0, Y and pairwise terms of the chunk's tokens;
* the gradient at the chunk start, through the chunk's tokens:
  D[n, 0] Y + Dout^T diag(D[., 0]) Q - Ddelta^T diag(D[., 0] beta) K.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def _decays(a: np.ndarray) -> np.ndarray:
    """D[t, s] = prod_{r=s+1..t} a_r for 0 <= s <= t <= n (tokens 1..n), 0 elsewhere."""
    n = a.shape[0]
    D = np.zeros((n + 1, n + 1), dtype=a.dtype)
    for s in range(n + 1):
        D[s, s] = 1.0
        for t in range(s + 1, n + 1):
            D[t, s] = D[t - 1, s] * a[t - 1]
    return D


def chunk_backward(S0, Y, q, k, v, a, b, dO, dtype=np.float64):
    """One chunk (n tokens, arrays [n, d]) from start state S0 [dv, dk] and end
    gradient Y [dv, dk].  Returns (dq, dk, dv, dalpha, dbeta, gradient at the
    chunk start, end state).  ``dtype`` is the arithmetic type (float64; a
    float32 evaluation measures the form's rounding for an fp32 kernel)."""
    S0, Y, q, k, v, a, b, dO = (np.asarray(x, dtype) for x in (S0, Y, q, k, v, a, b, dO))
    n = q.shape[0]
    D = _decays(a).astype(dtype)
    Dt = D[1:, 1:]                 # D[t, s], t, s = 1..n
    g = D[1:, 0]                   # D[t, 0]
    gp = D[:-1, 0]                 # D[t-1, 0]
    Dp = D[:-1, 1:]                # Dp[t, r] = D[t-1, r] (nonzero for r < t)
    dn = D[n, 1:]                  # D[n, t]
    KK, KQ = k @ k.T, k @ q.T
    lower = np.tril(np.ones((n, n), dtype), -1)
    A = b[:, None] * Dt * KK * lower
    Delta = solve_triangular(np.eye(n, dtype=dtype) + A, b[:, None] * (v - g[:, None] * (k @ S0.T)), lower=True,
                             unit_diagonal=True).astype(dtype)
    U = gp[:, None] * (k @ S0.T) + (Dp * KK.T * lower) @ Delta           # u_t = S_{t-1} k_t
    S_end = D[n, 0] * S0 + (dn[:, None] * Delta).T @ k
    # backward substitution for ddelta
    M = Dt.T * KQ * np.triu(np.ones((n, n), dtype))                       # M[t, s] = D[s, t] (k_t . q_s), s >= t
    rhs = dn[:, None] * (k @ Y.T) + M @ dO
    Dd = solve_triangular(np.eye(n, dtype=dtype) + A.T, rhs, lower=False, unit_diagonal=True).astype(dtype)
    dv = b[:, None] * Dd
    dbeta = np.sum(Dd * (v - a[:, None] * U), axis=1)
    DoDel = dO @ Delta.T                                                  # [t, r] = dO_t . delta_r
    incl = np.tril(np.ones((n, n), dtype))
    dq = g[:, None] * (dO @ S0) + (Dt * DoDel * incl) @ k
    DelDo = DoDel.T                                                       # [t, s] = delta_t . dO_s
    DelDd = Delta @ Dd.T                                                  # [t, s] = delta_t . ddelta_s
    upper_incl = np.triu(np.ones((n, n), dtype))
    upper = np.triu(np.ones((n, n), dtype), 1)
    dk = (dn[:, None] * (Delta @ Y) + (Dt.T * DelDo * upper_incl) @ q
          - (Dt.T * DelDd * upper * b[None, :]) @ k
          - (a * b)[:, None] * (gp[:, None] * (Dd @ S0) + (Dp * DelDd.T * lower) @ k))
    # dalpha: <H_t, S_{t-1}> expanded
    YS = np.sum(Y * S0)
    av = np.sum((dO @ S0) * q, axis=1)          # dO_s^T S0 q_s
    bv = np.sum((Dd @ S0) * k, axis=1)          # ddelta_s^T S0 k_s
    cv = np.sum((Delta @ Y) * k, axis=1)        # delta_r^T Y k_r
    E1 = DelDo * KQ                             # (delta_r . dO_s)(k_r . q_s)
    E2 = DelDd * KK                             # (delta_r . ddelta_s)(k_r . k_s)
    dalpha = np.zeros(n, dtype)
    for t in range(n):
        w_ge = Dt[t:, t]                                      # D[s, t] for s >= t
        w_gt = Dt[t + 1:, t] * b[t + 1:]                      # D[s, t] beta_s for s > t
        psi = gp[t] * (dn[t] * YS + w_ge @ av[t:] - w_gt @ bv[t + 1:])
        if t > 0:
            wr = Dp[t, :t]                                    # D[t-1, r] for r < t
            psi += wr @ (dn[t] * cv[:t] + E1[:t, t:] @ w_ge - E2[:t, t + 1:] @ w_gt)
        dalpha[t] = psi - b[t] * (Dd[t] @ U[t])
    G0 = D[n, 0] * Y + (g[:, None] * dO).T @ q - ((g * b)[:, None] * Dd).T @ k
    return dq, dk, dv, dalpha, dbeta, G0, S_end


def adjoint(q, k, v, alpha, beta, dO, cu_seqlens, C, state_in=None, dstate_out=None, dtype=np.float64):
    """Gradient of sum dO . o (+ <dstate_out, final state>) per sequence and
    head, chunk by chunk, in ``dtype`` arithmetic (fp64 by default).  Same
    layouts and results as oracle.adjoint."""
    q, k, v, dO = (np.asarray(x, np.float64) for x in (q, k, v, dO))
    alpha, beta = np.asarray(alpha, np.float64), np.asarray(beta, np.float64)
    cu = np.asarray(cu_seqlens)
    T, H, dk_ = k.shape
    dv_ = v.shape[2]
    N = len(cu) - 1
    out = dict(dq=np.zeros((T, H, dk_)), dk=np.zeros((T, H, dk_)), dv=np.zeros((T, H, dv_)),
               dalpha=np.zeros((T, H)), dbeta=np.zeros((T, H)), dstate_in=np.zeros((N, H, dv_, dk_)))
    for n in range(N):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        spans = [(s, min(s + C, t1)) for s in range(t0, t1, C)]
        for h in range(H):
            S = np.zeros((dv_, dk_)) if state_in is None else np.asarray(state_in, np.float64)[n, h].copy()
            starts = []
            for s0, s1 in spans:          # forward: the state at every chunk start
                starts.append(S)
                *_, S = chunk_backward(S, np.zeros((dv_, dk_)), q[s0:s1, h], k[s0:s1, h], v[s0:s1, h],
                                       alpha[s0:s1, h], beta[s0:s1, h], dO[s0:s1, h], dtype)
            Y = np.zeros((dv_, dk_)) if dstate_out is None else np.asarray(dstate_out, np.float64)[n, h].copy()
            for (s0, s1), S0 in reversed(list(zip(spans, starts))):
                dq, dkk, dvv, da, db, Y, _ = chunk_backward(S0, Y, q[s0:s1, h], k[s0:s1, h], v[s0:s1, h],
                                                            alpha[s0:s1, h], beta[s0:s1, h], dO[s0:s1, h], dtype)
                out["dq"][s0:s1, h], out["dk"][s0:s1, h], out["dv"][s0:s1, h] = dq, dkk, dvv
                out["dalpha"][s0:s1, h], out["dbeta"][s0:s1, h] = da, db
            out["dstate_in"][n, h] = Y
    return out
