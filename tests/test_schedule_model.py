"""Pins of the fp32 schedule model (CPU only).

The C schedule model is the bit pattern the CUDA kernels must reproduce.
It is pinned by: an exact-rational replay of the schedule with explicit
binary32 rounding (oracle.exact), a golden worked trace, the fp64 oracle
within tolerance, and the CPR self-consistency properties (prefill equals
decode, split equals unsplit, batch invariance) bit for bit.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import exact
from gated_deltanet_cpr_delta_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "schedule_trace_T3_d8.txt")


# ------------------------------------------------------------------ rn32 pins
def test_rn32_matches_numpy_cast(rng):
    xs = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-40, 38, 2000),
                         rng.standard_normal(200) * 1e-42])
    for x in xs:
        assert exact.rn32(Fraction(float(x))) == Fraction(float(np.float32(x)))


def test_rn32_ties_and_subnormals():
    tiny = Fraction(1, 2 ** 149)
    assert exact.rn32(tiny) == tiny
    assert exact.rn32(tiny / 2) == 0                  # tie -> even (0)
    assert exact.rn32(3 * tiny / 2) == 2 * tiny       # tie -> even (2)
    assert exact.rn32(1 + Fraction(1, 2 ** 24)) == 1  # tie -> even
    assert exact.rn32(1 + Fraction(3, 2 ** 24)) == 1 + Fraction(2, 2 ** 23)
    with pytest.raises(OverflowError):
        exact.rn32(Fraction(2) ** 128)


def _as_frac(a):
    return [[Fraction(float(x)) for x in row] for row in a]


@pytest.mark.parametrize("T,dk,dv,C,seed,folds", [(5, 8, 3, 2, 0, False), (9, 16, 2, 4, 1, False),
                                                   (7, 8, 4, 3, 2, False), (9, 8, 3, 9, 3, True)])
def test_c_model_equals_exact_rounding_replay(T, dk, dv, C, seed, folds):
    b = synth.make_batch(seed, [T], 1, dk, dv, "f32")
    if folds:  # decays that push the running scale below 2^-64 (folds), and a reset
        b.alpha[1, 0] = np.float32(2.0 ** -40)
        b.alpha[2, 0] = np.float32(2.0 ** -30)   # scale 2^-70 -> fold
        b.alpha[4, 0] = 0.0                      # reset -> fold
        b.alpha[6, 0] = np.float32(3e-38)        # -> fold
    S0 = synth.bf16_values(np.random.default_rng(seed).standard_normal((1, 1, dv, dk)).astype(np.float32))
    m = oracle.schedule_forward(b.q, b.k, b.v, b.alpha, b.beta, b.cu_seqlens, C, S0)
    sch = exact.Fp32Schedule()
    o, states = sch.forward(_as_frac(b.q[:, 0]), _as_frac(b.k[:, 0]), _as_frac(b.v[:, 0]),
                            [Fraction(float(x)) for x in b.alpha[:, 0]],
                            [Fraction(float(x)) for x in b.beta[:, 0]], C, _as_frac(S0[0, 0]))
    assert np.array_equal(m["o"][:, 0], np.array([[float(x) for x in r] for r in o], np.float32))
    for s, S in enumerate(states):
        assert np.array_equal(m["states"][s, 0], np.array([[float(x) for x in r] for r in S], np.float32))


def _read_golden():
    rows = {}
    for line in open(GOLDEN):
        if line.startswith("#"):
            continue
        parts = line.split()
        if parts[0] in ("alpha", "beta"):
            rows[parts[0]] = [float.fromhex(x) for x in parts[1:]]
        elif parts[0] == "state":
            rows.setdefault("state", {})[(int(parts[1]), int(parts[2]))] = [float.fromhex(x) for x in parts[3:]]
        else:
            rows.setdefault(parts[0], {})[int(parts[1])] = [float.fromhex(x) for x in parts[2:]]
    return rows


def test_c_model_matches_golden_trace():
    g = _read_golden()
    T = 3
    q = np.array([g["q"][t] for t in range(T)], np.float32)[:, None, :]
    k = np.array([g["k"][t] for t in range(T)], np.float32)[:, None, :]
    v = np.array([g["v"][t] for t in range(T)], np.float32)[:, None, :]
    a = np.array(g["alpha"], np.float32)[:, None]
    b = np.array(g["beta"], np.float32)[:, None]
    m = oracle.schedule_forward(q, k, v, a, b, np.array([0, T], np.int32), 2)
    assert np.array_equal(m["o"][:, 0], np.array([g["o"][t] for t in range(T)], np.float32))
    for s in range(2):
        S = np.array([g["state"][(s, i)] for i in range(2)], np.float32)
        assert np.array_equal(m["states"][s, 0], S)
    # token 0 by hand: zero state, so delta = beta*v and o = beta*(k.q)*v
    assert m["o"][0, 0, 0] == np.float32(0.125) and m["o"][0, 0, 1] == np.float32(-0.25)


# ---------------------------------------------------- tolerance vs fp64 oracle
@pytest.mark.parametrize("dtype,dk,dv,C", [("f32", 32, 16, 16), ("bf16", 64, 32, 32), ("f32", 16, 16, 16)])
def test_model_within_tolerance_of_oracle(dtype, dk, dv, C):
    b = synth.make_batch(11, [300, C, 1, 2 * C + 3], 2, dk, dv, dtype)
    m = oracle.schedule_forward(b.q, b.k, b.v, b.alpha, b.beta, b.cu_seqlens, C)
    r = oracle.recurrent(b.q, b.k, b.v, b.alpha, b.beta, b.cu_seqlens, C)
    err = np.max(np.abs(m["o"].astype(np.float64) - r["o"]))
    serr = np.max(np.abs(m["states"].astype(np.float64) - r["states"]))
    if dtype == "f32":
        assert err <= 1e-4 and serr <= 1e-4
    else:
        # the model's fp32 output; the bf16 cast adds at most 2^-9 relative
        assert err <= 2e-2 * np.max(np.abs(r["o"]))
        assert serr <= 2e-2 * np.max(np.abs(r["states"]))


# ----------------------------------------------------- CPR self-consistency
def _decode_from(bat, Lp, C, steps):
    """Prefill the first Lp tokens of every sequence, then decode `steps` tokens."""
    N = len(bat.lengths)
    pre = bat.subset(range(N))
    cu = bat.cu_seqlens
    sl = np.concatenate([np.arange(cu[n], cu[n] + Lp) for n in range(N)])
    cu_p = (np.arange(N + 1) * Lp).astype(np.int32)
    m = oracle.schedule_forward(pre.q[sl], pre.k[sl], pre.v[sl], pre.alpha[sl], pre.beta[sl], cu_p, C,
                                with_cache=True)
    outs = []
    for s in range(steps):
        idx = cu[:-1] + Lp + s
        outs.append(oracle.schedule_decode_step(m, bat.q[idx], bat.k[idx], bat.v[idx],
                                                bat.alpha[idx], bat.beta[idx], C))
    return m, outs


@pytest.mark.parametrize("Lp,steps,C", [(0, 40, 16), (32, 37, 16), (21, 30, 8)])
def test_prefill_equals_decode_bitwise(Lp, steps, C):
    N, H, dk, dv = 3, 2, 16, 8
    bat = synth.make_batch(5, [Lp + steps] * N, H, dk, dv, "bf16")
    full = oracle.schedule_forward(bat.q, bat.k, bat.v, bat.alpha, bat.beta, bat.cu_seqlens, C,
                                   with_cache=True)
    m, outs = _decode_from(bat, Lp, C, steps)
    for s in range(steps):
        idx = bat.cu_seqlens[:-1] + Lp + s
        assert np.array_equal(outs[s], full["o"][idx]), s
    for key in ("S_b", "R", "rscale", "pos", "kbuf", "vbuf", "abuf", "bbuf"):
        if key in ("kbuf", "vbuf", "abuf", "bbuf"):
            p = int(full["pos"][0, 0])
            assert np.array_equal(m[key][:, :, :p], full[key][:, :, :p]), key
        else:
            assert np.array_equal(m[key], full[key]), key
    # the boundary states seen by decode are the prefill's chunk states
    L = Lp + steps
    last = np.cumsum([L // C + 1] * N) - 1
    assert np.array_equal(m["S_b"], full["states"][last])


def test_tok_from_states_reproduces_the_model_forward():
    """Driving the model's P_tok from given boundary states (its own here)
    reproduces its forward outputs and running states bit for bit."""
    C = 16
    bat = synth.make_batch(10, [40, 16, 5, 0, 33], 2, 16, 16, "bf16")
    m = oracle.schedule_forward(bat.q, bat.k, bat.v, bat.alpha, bat.beta, bat.cu_seqlens, C, with_cache=True)
    o, Rf, Rs = oracle.schedule_tok_from_states(bat.q, bat.k, bat.v, bat.alpha, bat.beta, m["states"],
                                                bat.cu_seqlens, C)
    assert np.array_equal(o, m["o"]) and np.array_equal(Rf, m["R"]) and np.array_equal(Rs, m["rscale"])
    # and it really uses the states it is given: other states change the outputs
    o2, _, _ = oracle.schedule_tok_from_states(bat.q, bat.k, bat.v, bat.alpha, bat.beta, m["states"] * 2,
                                               bat.cu_seqlens, C)
    assert not np.array_equal(o2, m["o"])


def test_split_at_chunk_boundary_equals_unsplit():
    C, L = 16, 100
    bat = synth.make_batch(6, [L], 2, 16, 16, "bf16")
    full = oracle.schedule_forward(bat.q, bat.k, bat.v, bat.alpha, bat.beta, bat.cu_seqlens, C)
    for a in (16, 48, 96):
        p1 = oracle.schedule_forward(bat.q[:a], bat.k[:a], bat.v[:a], bat.alpha[:a], bat.beta[:a],
                                     np.array([0, a], np.int32), C)
        S_a = p1["states"][-1:]
        p2 = oracle.schedule_forward(bat.q[a:], bat.k[a:], bat.v[a:], bat.alpha[a:], bat.beta[a:],
                                     np.array([0, L - a], np.int32), C, state_in=S_a)
        assert np.array_equal(np.concatenate([p1["o"], p2["o"]]), full["o"])
        assert np.array_equal(np.concatenate([p1["states"], p2["states"][1:]]), full["states"])


def test_model_batch_invariance():
    C = 16
    bat = synth.make_batch(8, [50, 16, 3, 77], 2, 16, 8, "bf16")
    full = oracle.schedule_forward(bat.q, bat.k, bat.v, bat.alpha, bat.beta, bat.cu_seqlens, C)
    for n in range(4):
        one = bat.subset([n])
        r = oracle.schedule_forward(one.q, one.k, one.v, one.alpha, one.beta, one.cu_seqlens, C)
        a0, a1 = bat.cu_seqlens[n], bat.cu_seqlens[n + 1]
        assert np.array_equal(r["o"], full["o"][a0:a1])
        s0 = sum(int(L) // C + 1 for L in bat.lengths[:n])
        assert np.array_equal(r["states"], full["states"][s0:s0 + int(bat.lengths[n]) // C + 1])


def test_perturbed_schedule_is_detected_but_within_tolerance():
    """A schedule with one tree level swapped gives different bits (the
    bitwise checks can see it) while staying within the oracle tolerance."""

    class Swapped(exact.Fp32Schedule):
        def tree(self, x, y):
            L = len(x) // 8
            p = []
            for l in range(8):
                acc = self.mul(x[l * L], y[l * L])
                for m in range(1, L):
                    acc = self.fma(x[l * L + m], y[l * L + m], acc)
                p.append(acc)
            add = self.add
            return add(add(add(p[0], p[2]), add(p[1], p[3])), add(add(p[4], p[6]), add(p[5], p[7])))

    b = synth.make_batch(9, [12], 1, 16, 4, "f32")
    args = (_as_frac(b.q[:, 0]), _as_frac(b.k[:, 0]), _as_frac(b.v[:, 0]),
            [Fraction(float(x)) for x in b.alpha[:, 0]], [Fraction(float(x)) for x in b.beta[:, 0]], 4)
    o_a, _ = exact.Fp32Schedule().forward(*args)
    o_b, _ = Swapped().forward(*args)
    A = np.array([[float(x) for x in r] for r in o_a])
    B = np.array([[float(x) for x in r] for r in o_b])
    assert not np.array_equal(A, B)
    assert np.max(np.abs(A - B)) <= 1e-5


def test_scaled_state_folds_and_represents_the_state():
    """The running state is c * R.  A decay that would take the scale below
    2^-64 is folded into R (c returns to 1); alpha = 0 folds to an exact reset
    (R = beta v k^T, the closed form); and c * R stays within fp32 rounding of
    the plain recurrence's state in between."""
    dk, dv, C = 16, 8, 64
    b = synth.make_batch(21, [40], 1, dk, dv, "f32")
    b.alpha[5:10, 0] = np.float32(2.0 ** -20)   # four of these reach 2^-80: one fold
    b.alpha[20, 0] = 0.0                         # reset
    m = oracle.schedule_forward(b.q, b.k, b.v, b.alpha, b.beta, b.cu_seqlens, C, with_cache=True)
    R, Rs = m["R"][0, 0].astype(np.float64), float(m["rscale"][0, 0])
    r = oracle.recurrent(b.q, b.k, b.v, b.alpha, b.beta, b.cu_seqlens, C)
    # the running state after the last token (the 40 tokens are one partial chunk)
    Sref = np.zeros((dv, dk))
    for t in range(40):
        k, v, a, bb = b.k[t, 0].astype(np.float64), b.v[t, 0].astype(np.float64), float(b.alpha[t, 0]), float(b.beta[t, 0])
        Sref = a * (Sref - bb * np.outer(Sref @ k, k)) + bb * np.outer(v, k)
    assert np.max(np.abs(Rs * R - Sref)) <= 1e-5 * max(1.0, np.max(np.abs(Sref)))
    assert Rs <= 1.0 and Rs >= 2.0 ** -64
    # the scale after the last token is the product of the decays since the last fold (the reset)
    expect = np.float32(1.0)
    for t in range(21, 40):
        expect = np.float32(expect * b.alpha[t, 0])
    assert np.float32(Rs) == expect
    # the token after the reset sees only itself: o_20 = beta v (k . q) up to rounding
    t = 20
    o20 = float(b.beta[t, 0]) * b.v[t, 0].astype(np.float64) * float(b.k[t, 0].astype(np.float64) @ b.q[t, 0])
    assert np.max(np.abs(m["o"][t, 0] - o20)) <= 1e-6
    assert np.max(np.abs(m["o"] - r["o"])) <= 1e-5
