"""Writes tests/golden/schedule_trace_T3_d8.txt (run from the repo root).

A tiny worked trace of the fp32 CPR schedule: one sequence, one head,
T = 3 tokens, d_k = 8 (one element per leaf), d_v = 2, C = 2, so the trace
covers two P_tok steps, one P_chunk boundary update and one P_tok step
from the new boundary.  Every value is computed by oracle.exact's
Fp32Schedule (exact rationals rounded to binary32 after each operation);
inputs are small dyadic numbers so the trace can be followed by hand.
Values are written as Python float.hex() strings.
"""
import os
import sys
from fractions import Fraction as Fr

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
from oracle.exact import Fp32Schedule  # noqa: E402

q = [[Fr(1, 2), 0, Fr(-1, 4), 0, 0, Fr(1, 8), 0, Fr(3, 4)],
     [0, 1, 0, Fr(-1, 2), 0, 0, Fr(1, 4), 0],
     [Fr(1, 4)] * 8]
k = [[Fr(1, 2), Fr(1, 2), 0, 0, Fr(1, 2), 0, Fr(-1, 2), 0],
     [0, Fr(3, 4), Fr(1, 4), 0, 0, Fr(-1, 2), 0, Fr(1, 8)],
     [Fr(1, 3), 0, 0, Fr(1, 3), 0, 0, Fr(1, 3), 0]]
v = [[1, -2], [Fr(1, 3), Fr(5, 7)], [Fr(-3, 2), Fr(1, 10)]]
alpha = [Fr(3, 4), Fr(9, 10), Fr(1, 2)]
beta = [Fr(1, 2), Fr(1, 3), Fr(7, 8)]

sch = Fp32Schedule()
# inputs must themselves be binary32 values
from oracle.exact import rn32  # noqa: E402
q = [[rn32(x) for x in r] for r in q]
k = [[rn32(x) for x in r] for r in k]
v = [[rn32(x) for x in r] for r in v]
alpha = [rn32(x) for x in alpha]
beta = [rn32(x) for x in beta]
o, states = sch.forward(q, k, v, alpha, beta, C=2)

out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "schedule_trace_T3_d8.txt")
with open(out, "w") as f:
    f.write("# fp32 CPR schedule trace: T=3, d_k=8, d_v=2, C=2, zero initial state.\n")
    f.write("# Written by tests/golden/make_schedule_trace.py from oracle.exact.Fp32Schedule.\n")
    f.write("# Method: gated delta rule, chunkwise-parallel recurrent evaluation (IsoExec\n")
    f.write("# summary page, section 'Chunkwise-Parallel Recurrent (CPR) Gated DeltaNet').\n")
    for name, arr in (("q", q), ("k", k), ("v", v)):
        for t, row in enumerate(arr):
            f.write(f"{name} {t} " + " ".join(float(x).hex() for x in row) + "\n")
    f.write("alpha " + " ".join(float(x).hex() for x in alpha) + "\n")
    f.write("beta " + " ".join(float(x).hex() for x in beta) + "\n")
    for t, row in enumerate(o):
        f.write(f"o {t} " + " ".join(float(x).hex() for x in row) + "\n")
    for s, S in enumerate(states):
        for i, row in enumerate(S):
            f.write(f"state {s} {i} " + " ".join(float(x).hex() for x in row) + "\n")
print(out)
