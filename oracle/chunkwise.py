"""Chunkwise fp64 form of the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's cpu_baseline leg may
import this module.

The second, independent oracle form.  Chunkwise-parallel evaluation of
linear-attention layers is what the IsoExec commentary blog (section 10,
"Gated DeltaNet") describes as the training/prefill form; this is that form
for the gated delta rule, derived here from the recurrence
``S_t = alpha_t S_{t-1} + delta_t k_t^T``,
``delta_t = beta_t (v_t - alpha_t S_{t-1} k_t)``:

inside a chunk that starts from state S0, with decay products
``D[t,s] = alpha_{s+1} ... alpha_t`` (``D[t,t] = 1``), the deltas solve the
unit lower-triangular system

    (I + diag(beta) * strictly_lower(D o K K^T)) Delta
        = diag(beta) (V - diag(D[:,0]) K S0^T),

and then

    o_t   = D[t,0] S0 q_t + sum_{s<=t} D[t,s] (k_s . q_t) delta_s,
    S_end = D[n,0] S0 + sum_s D[n,s] delta_s k_s^T.

It uses a library triangular solve and dense numpy products in fp64 and
shares no code with the recurrent oracle.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def _decay_products(alpha_c: np.ndarray) -> np.ndarray:
    """D[t, s] = prod_{r=s+1..t} alpha_r for 0 <= s <= t <= n (tokens 1..n)."""
    n = alpha_c.shape[0]
    D = np.zeros((n + 1, n + 1), dtype=np.float64)
    for s in range(n + 1):
        D[s, s] = 1.0
        for t in range(s + 1, n + 1):
            D[t, s] = D[t - 1, s] * alpha_c[t - 1]
    return D


def chunk_step(S0, q_c, k_c, v_c, alpha_c, beta_c):
    """One chunk of n tokens from state S0 [dv, dk]: returns (O [n, dv], S_end)."""
    n = k_c.shape[0]
    D = _decay_products(alpha_c)
    Dts = D[1:, 1:]                       # token-token decays, t,s in 1..n
    Dt0 = D[1:, 0]                        # decay from the chunk start
    KK = k_c @ k_c.T
    A = np.eye(n) + beta_c[:, None] * np.tril(Dts * KK, k=-1)
    rhs = beta_c[:, None] * (v_c - Dt0[:, None] * (k_c @ S0.T))
    Delta = solve_triangular(A, rhs, lower=True, unit_diagonal=False)
    QK = q_c @ k_c.T                      # [t, s] = q_t . k_s
    O = Dt0[:, None] * (q_c @ S0.T) + np.tril(Dts * QK) @ Delta
    S_end = D[n, 0] * S0 + Delta.T @ (D[n, 1:][:, None] * k_c)
    return O, S_end


def forward(q, k, v, alpha, beta, cu_seqlens, C, state_in=None):
    """Chunkwise fp64 evaluation over a packed varlen batch.

    q, k [T, H, dk]; v [T, H, dv]; alpha, beta [T, H]; cu_seqlens [N+1].
    Returns dict(o [T,H,dv], states [sum(L//C+1), H, dv, dk], final [N,H,dv,dk]).
    """
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
    alpha = np.asarray(alpha, np.float64); beta = np.asarray(beta, np.float64)
    cu = np.asarray(cu_seqlens, np.int64)
    T, H, dk = k.shape
    dv = v.shape[2]
    N = cu.shape[0] - 1
    o = np.zeros((T, H, dv))
    nst = int(sum((cu[i + 1] - cu[i]) // C + 1 for i in range(N)))
    states = np.zeros((nst, H, dv, dk))
    final = np.zeros((N, H, dv, dk))
    slot0 = 0
    for nseq in range(N):
        a0, L = int(cu[nseq]), int(cu[nseq + 1] - cu[nseq])
        for h in range(H):
            S = np.zeros((dv, dk)) if state_in is None else np.asarray(state_in, np.float64)[nseq, h].copy()
            slot = slot0
            states[slot, h] = S
            for c0 in range(0, L, C):
                sl = slice(a0 + c0, a0 + min(c0 + C, L))
                O, S = chunk_step(S, q[sl, h], k[sl, h], v[sl, h], alpha[sl, h], beta[sl, h])
                o[sl, h] = O
                if min(c0 + C, L) - c0 == C:
                    slot += 1
                    states[slot, h] = S
            final[nseq, h] = S
        slot0 += L // C + 1
    return dict(o=o, states=states, final=final)
