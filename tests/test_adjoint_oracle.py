"""Pins of the fp64 adjoint oracle (oracle/adjoint_fp64.c), the gradient of
L = sum_t dO_t . o_t through the gated delta rule.

* Complex-step derivatives: the recurrence is a polynomial in every input, so
  Im(L(x + i h e_j)) / h is the exact derivative up to rounding (no
  cancellation).  A complex128 forward written independently here, with the
  literal matrix (I - beta k k^T), gives every partial derivative on small
  inputs; the adjoint must match them all.
* A closed form: with alpha = 1 and beta = 0 the state never changes, so
  dq_t = S_0^T dO_t, dS_0 = sum_t dO_t q_t^T, dv = dk = 0 and
  dalpha_t = <sum_{t' >= t} dO_t' q_t'^T, S_0>.
* A gradient W for each final state (dstate_out) adds <W, S_final> to the
  loss: the complex-step check includes that term, and in the closed form
  W adds to dS_0 and to every G.
* Two independent forms agree: the token-by-token reverse sweep and the
  chunkwise form (oracle/chunkwise_adjoint.py: triangular solves and dense
  chunk products, no division by a gate), including alpha = 0 tokens.
"""
import numpy as np
import pytest

import oracle
from gated_deltanet_cpr_delta_b200 import synth


def _loss_complex(q, k, v, alpha, beta, S0, dO, cu, W=None):
    """sum_t dO_t . o_t (+ sum <W, S_final>) with the recurrence
    S_t = a S (I - b k k^T) + b v k^T, complex128."""
    L = 0.0 + 0.0j
    H = k.shape[1]
    for n in range(len(cu) - 1):
        for h in range(H):
            S = S0[n, h].astype(np.complex128).copy()
            for t in range(cu[n], cu[n + 1]):
                kt, qt, vt = k[t, h], q[t, h], v[t, h]
                M = np.eye(len(kt), dtype=np.complex128) - beta[t, h] * np.outer(kt, kt)
                S = alpha[t, h] * (S @ M) + beta[t, h] * np.outer(vt, kt)
                L += dO[t, h] @ (S @ qt)
            if W is not None:
                L += np.sum(W[n, h] * S)
    return L


@pytest.mark.parametrize("C,with_w", [(2, False), (4, False), (4, True)])
def test_adjoint_matches_complex_step_derivatives(C, with_w):
    rng = np.random.default_rng(5)
    lens, H, dk, dv = [7, 4], 1, 3, 2
    b = synth.make_batch(21, lens, H, dk, dv, "f32")
    T = int(b.cu_seqlens[-1])
    S0 = rng.standard_normal((2, H, dv, dk))
    dO = rng.standard_normal((T, H, dv))
    W = rng.standard_normal((2, H, dv, dk)) if with_w else None
    ins = dict(q=b.q.astype(np.float64), k=b.k.astype(np.float64), v=b.v.astype(np.float64),
               alpha=b.alpha.astype(np.float64), beta=b.beta.astype(np.float64), S0=S0)
    g = oracle.adjoint(ins["q"], ins["k"], ins["v"], ins["alpha"], ins["beta"], dO, b.cu_seqlens, C, state_in=S0,
                       dstate_out=W)
    grads = dict(q=g["dq"], k=g["dk"], v=g["dv"], alpha=g["dalpha"], beta=g["dbeta"], S0=g["dstate_in"])
    h = 1e-30
    for name, base in ins.items():
        for idx in np.ndindex(base.shape):
            x = {k_: v_.astype(np.complex128) for k_, v_ in ins.items()}
            x[name][idx] += 1j * h
            d = _loss_complex(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"], dO, b.cu_seqlens, W).imag / h
            assert abs(d - grads[name][idx]) <= 1e-12 * max(1.0, abs(d)), (name, idx, d, grads[name][idx])


def test_adjoint_closed_form_with_a_frozen_state():
    rng = np.random.default_rng(6)
    T, H, dk, dv = 9, 2, 4, 3
    q, k, v = (rng.standard_normal((T, H, d)) for d in (dk, dk, dv))
    alpha, beta = np.ones((T, H)), np.zeros((T, H))
    S0 = rng.standard_normal((1, H, dv, dk))
    dO = rng.standard_normal((T, H, dv))
    g = oracle.adjoint(q, k, v, alpha, beta, dO, np.array([0, T], np.int32), 4, state_in=S0)
    for h in range(H):
        assert np.allclose(g["dq"][:, h], dO[:, h] @ S0[0, h], rtol=0, atol=1e-12)
        assert np.allclose(g["dstate_in"][0, h], dO[:, h].T @ q[:, h], rtol=0, atol=1e-12)
        for t in range(T):
            Gt = dO[t:, h].T @ q[t:, h]
            assert abs(g["dalpha"][t, h] - np.sum(Gt * S0[0, h])) <= 1e-12 * max(1, abs(np.sum(Gt * S0[0, h])))
    assert np.all(g["dv"] == 0) and np.allclose(g["dk"], 0, atol=1e-14)


def test_adjoint_closed_form_frozen_state_with_final_gradient():
    rng = np.random.default_rng(16)
    T, H, dk, dv = 6, 2, 4, 3
    q, k, v = (rng.standard_normal((T, H, d)) for d in (dk, dk, dv))
    alpha, beta = np.ones((T, H)), np.zeros((T, H))
    S0 = rng.standard_normal((1, H, dv, dk))
    W = rng.standard_normal((1, H, dv, dk))
    dO = rng.standard_normal((T, H, dv))
    g = oracle.adjoint(q, k, v, alpha, beta, dO, np.array([0, T], np.int32), 4, state_in=S0, dstate_out=W)
    for h in range(H):
        assert np.allclose(g["dstate_in"][0, h], dO[:, h].T @ q[:, h] + W[0, h], rtol=0, atol=1e-12)
        for t in range(T):
            Gt = dO[t:, h].T @ q[t:, h] + W[0, h]
            assert abs(g["dalpha"][t, h] - np.sum(Gt * S0[0, h])) <= 1e-12 * max(1, abs(np.sum(Gt * S0[0, h])))
    # an empty sequence passes the final-state gradient straight through
    e = oracle.adjoint(q[:0], k[:0], v[:0], alpha[:0], beta[:0], dO[:0], np.array([0, 0], np.int32), 4,
                       dstate_out=W)
    assert np.array_equal(e["dstate_in"], W)


def test_adjoint_is_independent_of_the_checkpoint_span():
    b = synth.make_batch(22, [37, 1, 20], 2, 8, 4, "bf16")
    dO = np.random.default_rng(7).standard_normal((58, 2, 4))
    a = oracle.adjoint(b.q, b.k, b.v, b.alpha, b.beta, dO, b.cu_seqlens, 4)
    c = oracle.adjoint(b.q, b.k, b.v, b.alpha, b.beta, dO, b.cu_seqlens, 16)
    for key in a:
        assert np.allclose(a[key], c[key], rtol=1e-12, atol=1e-12), key


@pytest.mark.parametrize("C,lens,dt", [(4, [7, 4, 0], "f32"), (16, [37, 16, 5], "bf16"), (8, [20, 9], "f32")])
def test_chunkwise_adjoint_agrees_with_the_token_sweep(C, lens, dt):
    b = synth.make_batch(31, lens, 2, 8, 6, dt)
    rng = np.random.default_rng(C)
    T = b.q.shape[0]
    b.alpha[rng.choice(T, size=3, replace=False), 0] = 0.0   # resets
    b.beta[rng.choice(T, size=2, replace=False), 1] = 0.0
    b.beta[rng.choice(T, size=2, replace=False), 0] = 1.0
    S0 = rng.standard_normal((len(lens), 2, 6, 8)) * 0.3
    W = rng.standard_normal((len(lens), 2, 6, 8)) * 0.2
    dO = rng.standard_normal((T, 2, 6))
    r = oracle.adjoint(b.q, b.k, b.v, b.alpha, b.beta, dO, b.cu_seqlens, C, S0, dstate_out=W)
    c = oracle.adjoint_chunkwise(b.q, b.k, b.v, b.alpha, b.beta, dO, b.cu_seqlens, C, S0, dstate_out=W)
    for key in r:
        scale = max(np.max(np.abs(r[key])), 1e-12)
        assert np.max(np.abs(r[key] - c[key])) <= 1e-11 * scale, key


def test_chunkwise_adjoint_in_fp32_is_well_inside_the_backward_tolerance():
    """The chunk-level form evaluated in fp32 arithmetic (numpy float32, the
    same formulas), d = 128, C = 64, 1024 bf16-valued tokens: every gradient
    within 2e-6 of the fp64 token sweep, relative to its largest magnitude,
    100x inside the backward's 2e-4 bound.  A kernel with fp32-class products
    (3xTF32 on the tensor cores) evaluating this form meets the bound."""
    C, d, L = 64, 128, 1024
    b = synth.make_batch(4, [L], 1, d, d, "bf16")
    dO = synth.bf16_values(np.random.default_rng(7).standard_normal((L, 1, d)).astype(np.float32))
    r = oracle.adjoint(b.q, b.k, b.v, b.alpha, b.beta, dO, b.cu_seqlens, C)
    c = oracle.adjoint_chunkwise(b.q, b.k, b.v, b.alpha, b.beta, dO, b.cu_seqlens, C, dtype=np.float32)
    for key in r:
        scale = max(np.max(np.abs(r[key])), 1e-12)
        assert np.max(np.abs(r[key] - c[key].astype(np.float64))) <= 2e-6 * scale, key


def test_backward_chain_step_is_the_forward_chain_transposed():
    """The chunk-start gradient of the chunkwise adjoint equals
    gamma_n Y - (Y Kt^T) W + F_c with W = T diag(D[.,0] beta) K,
    Kt = diag(D[n,.]) K and F_c from the chunk's own inputs; the end state
    equals gamma_n S0 - (S0 W^T) Kt + U0^T Kt (the forward's update); and W,
    U0 are what the forward's chunk-local forward substitution produces."""
    from oracle import chunkwise_adjoint as ca
    rng = np.random.default_rng(41)
    n, dk, dv = 12, 8, 6
    q, k = rng.standard_normal((n, dk)), rng.standard_normal((n, dk))
    v, dO = rng.standard_normal((n, dv)), rng.standard_normal((n, dv))
    a, b = rng.uniform(0.3, 1.0, n), rng.uniform(0.0, 1.0, n)
    a[4] = 0.0
    S0, Y = rng.standard_normal((dv, dk)), rng.standard_normal((dv, dk))
    *_, G0, S_end = ca.chunk_backward(S0, Y, q, k, v, a, b, dO)
    D = ca._decays(a)
    g, dn, gn = D[1:, 0], D[n, 1:], D[n, 0]
    A = b[:, None] * D[1:, 1:] * (k @ k.T) * np.tril(np.ones((n, n)), -1)
    T = np.linalg.inv(np.eye(n) + A)
    W = T @ ((g * b)[:, None] * k)
    U0 = T @ (b[:, None] * v)
    Kt = dn[:, None] * k
    M = D[1:, 1:].T * (k @ q.T) * np.triu(np.ones((n, n)))
    F = dO.T @ (g[:, None] * q) - (T.T @ M @ dO).T @ ((g * b)[:, None] * k)
    assert np.allclose(G0, gn * Y - (Y @ Kt.T) @ W + F, rtol=0, atol=1e-12)
    assert np.allclose(S_end, gn * S0 - (S0 @ W.T) @ Kt + U0.T @ Kt, rtol=0, atol=1e-12)
    # W and U0 are the forward's chunk-local precompute, by its forward substitution:
    # w_t = beta_t (D[t,0] k_t - sum_{s<t} D[t,s] (k_s . k_t) w_s), u0_t likewise with v_t
    w, u0 = np.zeros((n, dk)), np.zeros((n, dv))
    for t in range(n):
        c = D[t + 1, 1:t + 1] * (k[:t] @ k[t])
        w[t] = b[t] * (D[t + 1, 0] * k[t] - c @ w[:t])
        u0[t] = b[t] * (v[t] - c @ u0[:t])
    assert np.allclose(w, W, rtol=0, atol=1e-12) and np.allclose(u0, U0, rtol=0, atol=1e-12)


def test_adjoint_forms_agree_on_random_shapes():
    """Property check over random small problems: lengths 0..20 (ragged, with
    empty sequences), C in {1, 2, 4, 8}, d_k, d_v in 2..4, gates with exact
    zeros and ones, random state_in and dstate_out.  The token sweep and the
    chunkwise form agree to 1e-10 relative on every gradient."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=40, deadline=None, derandomize=True)
    @given(st.integers(0, 2**31 - 1))
    def check(seed):
        rng = np.random.default_rng(seed)
        N, H = int(rng.integers(1, 4)), int(rng.integers(1, 3))
        dk, dv, C = int(rng.integers(2, 5)), int(rng.integers(2, 5)), int(rng.choice([1, 2, 4, 8]))
        lens = rng.integers(0, 21, N)
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        T = int(cu[-1])
        q, k = rng.standard_normal((T, H, dk)), rng.standard_normal((T, H, dk)) * 0.5
        v, dO = rng.standard_normal((T, H, dv)), rng.standard_normal((T, H, dv))
        alpha = rng.uniform(0.0, 1.0, (T, H))
        beta = rng.uniform(0.0, 1.0, (T, H))
        if T:
            alpha[rng.integers(0, T, 2), rng.integers(0, H, 2)] = 0.0
            beta[rng.integers(0, T, 2), rng.integers(0, H, 2)] = 1.0
        S0 = rng.standard_normal((N, H, dv, dk))
        W = rng.standard_normal((N, H, dv, dk))
        r = oracle.adjoint(q, k, v, alpha, beta, dO, cu, C, S0, dstate_out=W)
        c = oracle.adjoint_chunkwise(q, k, v, alpha, beta, dO, cu, C, S0, dstate_out=W)
        for key in r:
            scale = max(np.max(np.abs(r[key])) if r[key].size else 0.0, 1e-12)
            assert np.max(np.abs(r[key] - c[key]), initial=0.0) <= 1e-10 * scale, (seed, key)

    check()
