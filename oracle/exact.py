"""Exact-rational oracle pieces -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's cpu_baseline leg may
import this module.

* :func:`recurrence` evaluates the gated delta rule of the IsoExec summary
  page (section "Chunkwise-Parallel Recurrent (CPR) Gated DeltaNet") in
  exact rational arithmetic, forming ``I - beta k k^T`` literally:
  ``S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T``,
  ``o_t = S_t q_t``.  The rule uses only +, - and *, so every value is an
  exact rational when the inputs are.
* :func:`rn32` rounds an exact rational to the nearest IEEE binary32 value
  (ties to even, subnormals kept).  With it, :class:`Fp32Schedule` replays
  the written-down fp32 arithmetic schedule one rounded operation at a
  time; it is an independent check of the C schedule model, which uses
  hardware float arithmetic and libm ``fmaf``.
"""
from __future__ import annotations

from fractions import Fraction
from typing import List, Sequence

Mat = List[List[Fraction]]


def F(x) -> Fraction:
    """Exact rational value of a float (or int/Fraction)."""
    return x if isinstance(x, Fraction) else Fraction(x)


def recurrence(q, k, v, alpha, beta, S0=None):
    """Exact gated delta rule for ONE (sequence, head).

    q, k: T x d_k nested sequences; v: T x d_v; alpha, beta: length T;
    S0: d_v x d_k or None (zeros).  Returns (o [T][d_v], states [T+1]) with
    states[t] the exact state after t tokens (states[0] = S0).
    """
    T = len(k)
    dk = len(k[0]) if T else (len(S0[0]) if S0 else 0)
    dv = len(v[0]) if T else (len(S0) if S0 else 0)
    S = [[F(S0[i][j]) if S0 is not None else Fraction(0) for j in range(dk)] for i in range(dv)]
    states = [[row[:] for row in S]]
    outs = []
    for t in range(T):
        kt = [F(x) for x in k[t]]
        qt = [F(x) for x in q[t]]
        vt = [F(x) for x in v[t]]
        a, b = F(alpha[t]), F(beta[t])
        # M = I - b k k^T  (d_k x d_k), formed literally
        M = [[(Fraction(1) if i == j else Fraction(0)) - b * kt[i] * kt[j] for j in range(dk)]
             for i in range(dk)]
        SM = [[sum((S[i][m] * M[m][j] for m in range(dk)), Fraction(0)) for j in range(dk)]
              for i in range(dv)]
        S = [[a * SM[i][j] + b * vt[i] * kt[j] for j in range(dk)] for i in range(dv)]
        outs.append([sum((S[i][j] * qt[j] for j in range(dk)), Fraction(0)) for i in range(dv)])
        states.append([row[:] for row in S])
    return outs, states


# ---------------------------------------------------------------- binary32 rounding
_EMIN = -126          # smallest normal exponent of binary32
_P = 24               # significand bits
_MAX = (2 - Fraction(1, 2 ** 23)) * Fraction(2) ** 127


def _floor_log2(x: Fraction) -> int:
    """floor(log2(x)) for x > 0, exactly."""
    e = x.numerator.bit_length() - x.denominator.bit_length()
    # adjust so that 2^e <= x < 2^(e+1)
    while Fraction(2) ** e > x:
        e -= 1
    while Fraction(2) ** (e + 1) <= x:
        e += 1
    return e


def rn32(x) -> Fraction:
    """Round an exact rational to binary32, nearest-even; subnormals kept."""
    x = F(x)
    if x == 0:
        return Fraction(0)
    sgn = -1 if x < 0 else 1
    ax = -x if x < 0 else x
    e = max(_floor_log2(ax), _EMIN)
    quantum = Fraction(2) ** (e - (_P - 1))
    n = ax / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    r = fl * quantum
    if r > _MAX:
        raise OverflowError("binary32 overflow")
    return sgn * r


def is_f32(x) -> bool:
    """True when the rational x is exactly a binary32 value."""
    return rn32(x) == F(x)


class Fp32Schedule:
    """The fp32 CPR schedule, replayed with exact rationals and an explicit
    binary32 rounding after every operation (tiny inputs only).

    ``mul(a,b) = rn32(a*b)``, ``add``/``sub`` likewise, ``rcp(a) = rn32(1/a)``
    and ``fma(a,b,c) = rn32(a*b + c)`` (one rounding).  The reduction tree has
    NL = 8 contiguous leaves over d_k, each an ascending fused multiply-add
    chain started by a plain product, combined by the fixed tree
    ((0+1)+(2+3))+((4+5)+(6+7)).  The per-token step keeps its running state
    as a scale times a matrix (see :meth:`p_tok`).
    """

    #: a decay whose new scale would fall below this is folded into the matrix
    FOLD_TAU = Fraction(1, 2 ** 64)

    NL = 8

    @staticmethod
    def mul(a, b):
        return rn32(F(a) * F(b))

    @staticmethod
    def add(a, b):
        return rn32(F(a) + F(b))

    @staticmethod
    def sub(a, b):
        return rn32(F(a) - F(b))

    @staticmethod
    def fma(a, b, c):
        return rn32(F(a) * F(b) + F(c))

    def tree(self, x: Sequence, y: Sequence) -> Fraction:
        dk = len(x)
        assert dk % self.NL == 0
        L = dk // self.NL
        p = []
        for l in range(self.NL):
            acc = self.mul(x[l * L], y[l * L])
            for m in range(1, L):
                acc = self.fma(x[l * L + m], y[l * L + m], acc)
            p.append(acc)
        add = self.add
        return add(add(add(p[0], p[1]), add(p[2], p[3])), add(add(p[4], p[5]), add(p[6], p[7])))

    @staticmethod
    def rcp(a):
        return rn32(1 / F(a))

    def p_tok(self, R: Mat, c, k, v, q, a, b):
        """One per-token step on the running state c * R; returns (R, c, o).

        With cn = a*c: if cn >= 2^-64 the decay stays in the scale (c <- cn)
        and row i gets dt = (b*(v_i - cn*tree(R_i, k))) * rcp(cn),
        R_ij <- fma(dt, k_j, R_ij), o_i = cn * fma(dt, tree(k, q), tree(R_i, q));
        otherwise it is folded into R (c <- 1): d = b*(v_i - cn*tree(R_i, k)),
        R_ij <- fma(d, k_j, cn*R_ij), o_i = fma(d, tree(k, q), cn*tree(R_i, q)).
        The trees over R are taken before the update."""
        kq = self.tree(k, q)
        cn = self.mul(a, c)
        fold = not (cn >= self.FOLD_TAU)
        rc = None if fold else self.rcp(cn)
        R2, o = [], []
        for i, Ri in enumerate(R):
            dk = self.tree(Ri, k)
            dq = self.tree(Ri, q)
            d = self.mul(b, self.sub(v[i], self.mul(cn, dk)))
            if not fold:
                dt = self.mul(d, rc)
                R2.append([self.fma(dt, k[j], Ri[j]) for j in range(len(Ri))])
                o.append(self.mul(cn, self.fma(dt, kq, dq)))
            else:
                R2.append([self.fma(d, k[j], self.mul(cn, Ri[j])) for j in range(len(Ri))])
                o.append(self.fma(d, kq, self.mul(cn, dq)))
        return R2, (Fraction(1) if fold else cn), o

    def p_chunk(self, S: Mat, ks, vs, al, be):
        """Chunk-boundary update of S over the C tokens ks/vs/al/be."""
        C = len(ks)
        dk, dv = len(ks[0]), len(vs[0])
        D = [[None] * (C + 1) for _ in range(C + 1)]
        for s in range(C + 1):
            D[s][s] = Fraction(1)
            for t in range(s + 1, C + 1):
                D[t][s] = self.mul(D[t - 1][s], al[t - 1])
        c = {}
        for t in range(2, C + 1):
            for s in range(1, t):
                c[t, s] = self.mul(D[t][s], self.tree(ks[s - 1], ks[t - 1]))
        u0, w = {}, {}
        for t in range(1, C + 1):
            bt = be[t - 1]
            row = []
            for i in range(dv):
                acc = F(vs[t - 1][i])
                for s in range(1, t):
                    acc = self.fma(-c[t, s], u0[s][i], acc)
                row.append(self.mul(bt, acc))
            u0[t] = row
            row = []
            for j in range(dk):
                acc = self.mul(D[t][0], ks[t - 1][j])
                for s in range(1, t):
                    acc = self.fma(-c[t, s], w[s][j], acc)
                row.append(self.mul(bt, acc))
            w[t] = row
        e = {}
        for t in range(1, C + 1):
            e[t] = [self.mul(D[C][t], self.sub(u0[t][i], self.tree(S[i], w[t]))) for i in range(dv)]
        out = []
        for i in range(dv):
            row = []
            for j in range(dk):
                acc = self.mul(D[C][0], S[i][j])
                for t in range(1, C + 1):
                    acc = self.fma(e[t][i], ks[t - 1][j], acc)
                row.append(acc)
            out.append(row)
        return out

    def forward(self, q, k, v, alpha, beta, C, S0=None):
        """CPR forward for ONE (sequence, head): (o, boundary states)."""
        T = len(k)
        dk, dv = len(k[0]), len(v[0])
        B = [[F(S0[i][j]) if S0 is not None else Fraction(0) for j in range(dk)] for i in range(dv)]
        states = [B]
        outs = []
        for c0 in range(0, T, C):
            n = min(C, T - c0)
            R, c = B, Fraction(1)
            for t in range(c0, c0 + n):
                R, c, o = self.p_tok(R, c, k[t], v[t], q[t], alpha[t], beta[t])
                outs.append(o)
            if n == C:
                B = self.p_chunk(B, k[c0:c0 + C], v[c0:c0 + C], alpha[c0:c0 + C], beta[c0:c0 + C])
                states.append(B)
        return outs, states
