"""Pins of the fp64 oracle (CPU only).

Every check compares the oracle with something other than itself: exact
rational arithmetic, closed forms of the gated delta rule, an independent
chunkwise formulation, or structural invariants (batch composition,
affinity in the initial state).
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import exact
from gated_deltanet_cpr_delta_b200 import synth


def _rand_inputs(rng, T, H, dk, dv, unit=True):
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    if unit:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    a = np.exp(-np.logaddexp(0, rng.standard_normal((T, H))))
    b = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    return q, k, v, a, b


def _rec(q, k, v, a, b, cu, C, S0=None):
    return oracle.recurrent(q, k, v, a, b, np.asarray(cu, np.int32), C, S0)


@pytest.mark.parametrize("T,dk,dv,C", [(6, 3, 2, 2), (8, 4, 3, 4), (5, 2, 4, 3)])
def test_recurrent_matches_exact_rationals(rng, T, dk, dv, C):
    q, k, v, a, b = _rand_inputs(rng, T, 1, dk, dv, unit=False)
    S0 = rng.standard_normal((1, 1, dv, dk))
    out = _rec(q, k, v, a, b, [0, T], C, S0)
    eo, es = exact.recurrence(q[:, 0], k[:, 0], v[:, 0], a[:, 0], b[:, 0], S0[0, 0])
    o_ex = np.array([[float(x) for x in row] for row in eo])
    assert np.max(np.abs(out["o"][:, 0] - o_ex)) <= 1e-12 * max(1.0, np.max(np.abs(o_ex)))
    for slot, t in enumerate(range(0, T + 1, C)):
        s_ex = np.array([[float(x) for x in r] for r in es[t]])
        assert np.max(np.abs(out["states"][slot, 0] - s_ex)) <= 1e-12 * max(1.0, np.max(np.abs(s_ex)))
    f_ex = np.array([[float(x) for x in r] for r in es[T]])
    assert np.max(np.abs(out["final"][0, 0] - f_ex)) <= 1e-12 * max(1.0, np.max(np.abs(f_ex)))


def test_exact_recurrence_hand_example():
    # d_k = d_v = 1, two tokens, worked by hand:
    # S1 = a1*S0*(1 - b1 k1^2) + b1 v1 k1 = 1/2*2*(1-1/2*1) + 1/2*3*1 = 1/2 + 3/2 = 2
    # o1 = S1 q1 = 2*2 = 4
    # S2 = a2*S1*(1 - b2 k2^2) + b2 v2 k2 = 1*2*(1 - 1/4*4) + 1/4*5*2 = 0 + 5/2
    # o2 = 5/2 * (-1) = -5/2
    o, st = exact.recurrence([[2], [-1]], [[1], [2]], [[3], [5]], [Fraction(1, 2), 1],
                             [Fraction(1, 2), Fraction(1, 4)], [[2]])
    assert o == [[4], [Fraction(-5, 2)]]
    assert st[1] == [[2]] and st[2] == [[Fraction(5, 2)]]


def test_alpha1_beta0_keeps_state(rng):
    T, H, dk, dv = 37, 3, 16, 8
    q, k, v, a, b = _rand_inputs(rng, T, H, dk, dv)
    a[:] = 1.0
    b[:] = 0.0
    S0 = rng.standard_normal((1, H, dv, dk))
    out = _rec(q, k, v, a, b, [0, T], 8, S0)
    assert np.array_equal(out["final"], S0)
    for s in range(out["states"].shape[0]):
        assert np.array_equal(out["states"][s], S0[0])
    o_ref = np.einsum("hij,thj->thi", S0[0], q)
    assert np.allclose(out["o"], o_ref, rtol=0, atol=1e-13)


def test_beta1_unit_key_writes_value(rng):
    T, H, dk, dv = 50, 2, 16, 16
    q, k, v, a, b = _rand_inputs(rng, T, H, dk, dv)
    b[:] = 1.0
    S0 = rng.standard_normal((1, H, dv, dk))
    for t in range(1, T + 1):
        out = _rec(q[:t], k[:t], v[:t], a[:t], b[:t], [0, t], 1000, S0)
        Sk = np.einsum("hij,hj->hi", out["final"][0], k[t - 1])
        assert np.allclose(Sk, v[t - 1], rtol=0, atol=1e-12)


def test_alpha0_resets_state(rng):
    T, H, dk, dv = 20, 2, 8, 5
    q, k, v, a, b = _rand_inputs(rng, T, H, dk, dv)
    a[:] = 0.0
    S0 = rng.standard_normal((1, H, dv, dk))
    out = _rec(q, k, v, a, b, [0, T], 4, S0)
    # S_t = beta_t v_t k_t^T, o_t = beta_t (k_t . q_t) v_t
    o_ref = (b * np.einsum("thj,thj->th", k, q))[:, :, None] * v
    assert np.allclose(out["o"], o_ref, rtol=0, atol=1e-14)
    S_last = b[-1][:, None, None] * np.einsum("hi,hj->hij", v[-1], k[-1])
    assert np.allclose(out["final"][0], S_last, rtol=0, atol=1e-14)


def test_orthonormal_keys_are_a_memory(rng):
    dk = dv = 16
    T = 12
    q, k, v, a, b = _rand_inputs(rng, T, 1, dk, dv)
    a[:] = 1.0
    b[:] = 1.0
    k[:] = 0.0
    for t in range(T):
        k[t, 0, t] = 1.0
    out = _rec(q, k, v, a, b, [0, T], 4)
    S = out["final"][0, 0]
    for j in range(T):
        assert np.allclose(S[:, j], v[j, 0], rtol=0, atol=1e-15)
    for j in range(T, dk):
        assert np.all(S[:, j] == 0)


def test_scalar_case_is_first_order_linear_recurrence(rng):
    T = 200
    q, k, v, a, b = _rand_inputs(rng, T, 1, 1, 1, unit=False)
    s0 = 0.7
    out = _rec(q, k, v, a, b, [0, T], 1000, np.full((1, 1, 1, 1), s0))
    # s_t = A_t s_{t-1} + B_t with A_t = alpha_t (1 - beta_t k_t^2), B_t = beta_t v_t k_t
    A = a[:, 0] * (1 - b[:, 0] * k[:, 0, 0] ** 2)
    Bc = b[:, 0] * v[:, 0, 0] * k[:, 0, 0]
    # closed form: s_T = (prod A) s0 + sum_t (prod_{r>t} A_r) B_t
    tail = np.array([np.prod(A[t + 1:]) for t in range(T)])
    sT = np.prod(A) * s0 + np.sum(tail * Bc)
    assert abs(out["final"][0, 0, 0, 0] - sT) <= 1e-12 * max(1, abs(sT))
    # and every output o_t = s_t q_t
    s = np.array([np.prod(A[:t + 1]) * s0 + np.sum([np.prod(A[r + 1:t + 1]) * Bc[r] for r in range(t + 1)])
                  for t in range(T)])
    assert np.allclose(out["o"][:, 0, 0], s * q[:, 0, 0], rtol=1e-11, atol=1e-12)


def test_state_is_affine_in_initial_state(rng):
    T, H, dk, dv = 40, 2, 8, 6
    q, k, v, a, b = _rand_inputs(rng, T, H, dk, dv)
    S0 = rng.standard_normal((1, H, dv, dk))
    f0 = _rec(q, k, v, a, b, [0, T], 8)["final"]
    f1 = _rec(q, k, v, a, b, [0, T], 8, S0)["final"]
    f2 = _rec(q, k, v, a, b, [0, T], 8, 2 * S0)["final"]
    assert np.allclose(f2 - f0, 2 * (f1 - f0), rtol=0, atol=1e-12)
    # the S0-dependent part does not depend on v
    v2 = rng.standard_normal(v.shape)
    g0 = _rec(q, k, v2, a, b, [0, T], 8)["final"]
    g1 = _rec(q, k, v2, a, b, [0, T], 8, S0)["final"]
    assert np.allclose(g1 - g0, f1 - f0, rtol=0, atol=1e-12)


@pytest.mark.parametrize("C", [4, 16, 64])
def test_chunkwise_form_agrees_with_recurrence(rng, C):
    lens = [1, C - 1, C, C + 1, 3 * C + 5, 256]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, dk, dv = int(cu[-1]), 2, 16, 8
    q, k, v, a, b = _rand_inputs(rng, T, H, dk, dv)
    S0 = rng.standard_normal((len(lens), H, dv, dk)) * 0.3
    r = _rec(q, k, v, a, b, cu, C, S0)
    c = oracle.chunkwise(q, k, v, a, b, cu, C, S0)
    for key in ("o", "states", "final"):
        scale = max(1.0, np.max(np.abs(r[key])))
        assert np.max(np.abs(r[key] - c[key])) <= 1e-11 * scale, key


def test_chunkwise_alpha_zero_no_nan(rng):
    T, H, dk, dv, C = 33, 1, 8, 4, 8
    q, k, v, a, b = _rand_inputs(rng, T, H, dk, dv)
    a[::3] = 0.0
    r = _rec(q, k, v, a, b, [0, T], C)
    c = oracle.chunkwise(q, k, v, a, b, [0, T], C)
    assert np.all(np.isfinite(c["o"]))
    assert np.max(np.abs(r["o"] - c["o"])) <= 1e-12


def test_batch_composition_invariance(rng):
    b = synth.make_batch(7, [40, 17, 64, 3], 2, 16, 16, "f32")
    full = oracle.recurrent(b.q, b.k, b.v, b.alpha, b.beta, b.cu_seqlens, 16)
    perm = [2, 0, 3, 1]
    pb = b.subset(perm)
    pf = oracle.recurrent(pb.q, pb.k, pb.v, pb.alpha, pb.beta, pb.cu_seqlens, 16)
    for new_pos, old in enumerate(perm):
        a0, a1 = b.cu_seqlens[old], b.cu_seqlens[old + 1]
        p0, p1 = pb.cu_seqlens[new_pos], pb.cu_seqlens[new_pos + 1]
        assert np.array_equal(full["o"][a0:a1], pf["o"][p0:p1])
        assert np.array_equal(full["final"][old], pf["final"][new_pos])
    alone = b.subset([2])
    af = oracle.recurrent(alone.q, alone.k, alone.v, alone.alpha, alone.beta, alone.cu_seqlens, 16)
    assert np.array_equal(af["o"], full["o"][b.cu_seqlens[2]:b.cu_seqlens[3]])


def test_chunk_states_are_prefix_states(rng):
    T, H, dk, dv, C = 50, 2, 8, 8, 16
    q, k, v, a, b = _rand_inputs(rng, T, H, dk, dv)
    r = _rec(q, k, v, a, b, [0, T], C)
    for n in range(T // C + 1):
        p = _rec(q[:n * C], k[:n * C], v[:n * C], a[:n * C], b[:n * C], [0, n * C], C)
        assert np.array_equal(r["states"][n], p["final"][0])
