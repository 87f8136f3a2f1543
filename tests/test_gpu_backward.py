"""GPU parity of the CPR backward (gdn_cpr_backward, through the C ABI)
against the fp64 adjoint oracle (oracle/adjoint_fp64.c).

The loss is L = sum_t dO_t . o_t.  The kernels compute in fp32-class
arithmetic from inputs that both sides read as the same values (bf16 inputs
are widened exactly): the boundary adjoints by a serial fp32 scan, each
chunk's gradients by dense chunk-form products on the tensor cores with every
fp32 operand split into two tf32 parts (lo*hi + hi*lo + hi*hi).  The only
differences are rounding in the forward's boundary states, the adjoints and
those products.  Bound: max|g - g*| <= 2e-4 * max(||g*||_inf, 1e-3) for every
gradient (the chunk form evaluated in fp32 stays within 4e-7 of the fp64
sweep on these sizes; the bound leaves a wide margin, and plain tf32 products
would exceed it).
Also: repeats are bit-identical (no atomics), batch composition does not change
a sequence's gradients, and a sampled (sequence, head) at the trainer's full
size (B=2, H=32, T=8192, d=128, C=64, bf16) matches the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import bits, to_device
from gated_deltanet_cpr_delta_b200 import gdn, synth

pytestmark = pytest.mark.gpu

DEV = "cuda"
NAMES = ("dq", "dk", "dv", "dalpha", "dbeta", "dstate_in")
REL = 2e-4


def _dO(seed, T, H, dv, dtype):
    x = (np.random.default_rng(seed).standard_normal((T, H, dv)) * 0.5).astype(np.float32)
    return synth.bf16_values(x) if dtype == "bf16" else x


def run(b, C, S0, dO):
    d = to_device(b)
    S0d = None if S0 is None else torch.from_numpy(S0).to(DEV)
    _, st = gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"], C,
                                cu_seqlens_host=d["cu_host"], state_in=S0d, out_dtype=torch.float32)
    dOd = torch.from_numpy(dO).to(DEV).to(d["q"].dtype)
    g = gdn.gdn_cpr_backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], dOd, st, d["cu_seqlens"], C,
                             cu_seqlens_host=d["cu_host"])
    torch.cuda.synchronize()
    return [x.cpu().numpy() for x in g]


def check(got, ref, what=""):
    for name, g in zip(NAMES, got):
        r = ref[name]
        if r.size == 0:
            continue
        err = float(np.max(np.abs(g.astype(np.float64) - r)))
        scale = max(float(np.max(np.abs(r))), 1e-3)
        assert err <= REL * scale, (what, name, err, scale)


SHAPES = [(d, C) for d in (16, 32, 64, 128) for C in (16, 32, 64)]


@pytest.mark.parametrize("d,C", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_vs_adjoint_oracle(d, C, dtype):
    lens = [1, C - 1, C, 0, C + 1, 3 * C + 5] if d <= 64 else [C - 1, 2 * C + 3, 0, C, 9]
    H = 3 if d <= 64 else 2
    b = synth.make_batch(200 + d + C, lens, H, d, d, dtype)
    S0 = (np.random.default_rng(d + 7 * C).standard_normal((len(lens), H, d, d)) * 0.2).astype(np.float32)
    dO = _dO(d * C, b.q.shape[0], H, d, dtype)
    got = run(b, C, S0, dO)
    ref = oracle.adjoint(b.q, b.k, b.v, b.alpha, b.beta, dO, b.cu_seqlens, C, S0)
    check(got, ref, f"d={d} C={C} {dtype}")


def test_backward_zero_state_in_and_repeats_bitwise():
    b = synth.make_batch(31, [200, 64, 7], 4, 128, 128, "bf16")
    dO = _dO(5, b.q.shape[0], 4, 128, "bf16")
    g1 = run(b, 64, None, dO)
    g2 = run(b, 64, None, dO)
    for x, y in zip(g1, g2):
        assert np.array_equal(bits(x), bits(y))
    check(g1, oracle.adjoint(b.q, b.k, b.v, b.alpha, b.beta, dO, b.cu_seqlens, 64), "zero state")


def test_backward_batch_composition_invariance():
    lens = [130, 64, 1, 77]
    b = synth.make_batch(41, lens, 2, 64, 64, "f32")
    dO = _dO(9, b.q.shape[0], 2, 64, "f32")
    g = run(b, 32, None, dO)
    # sequence 2 alone, then packed in another order
    cu = b.cu_seqlens
    for order in ([2], [3, 2, 0]):
        sub = b.subset(order)
        dsub = np.concatenate([dO[cu[s]:cu[s + 1]] for s in order])
        gs = run(sub, 32, None, dsub)
        off = 0
        for i, s in enumerate(order):
            L = lens[s]
            for name, a, c in zip(NAMES[:5], g[:5], gs[:5]):
                assert np.array_equal(bits(a[cu[s]:cu[s + 1]]), bits(c[off:off + L])), (order, s, name)
            assert np.array_equal(bits(g[5][s]), bits(gs[5][i]))
            off += L


def test_backward_empty_batches():
    b = synth.make_batch(3, [0, 0], 2, 32, 32, "f32")
    g = run(b, 16, None, np.zeros((0, 2, 32), np.float32))
    assert g[0].shape == (0, 2, 32)
    assert np.array_equal(g[5], np.zeros((2, 2, 32, 32), np.float32))


def test_backward_trainer_size_sampled_head_vs_oracle():
    """Full trainer size; one (sequence, head) pair compared with the oracle
    (heads and sequences are independent, so the sample is exact)."""
    cfg = synth.TRAIN
    B, H, T, d, C = cfg["B"], cfg["H"], cfg["T"], cfg["dk"], cfg["C"]
    bd = synth.make_batch_device(cfg["seed"], [T] * B, H, d, d, cfg["dtype"])
    q, k, v, alpha, beta, cu = (bd[x] for x in ("q", "k", "v", "alpha", "beta", "cu_seqlens"))
    g = torch.Generator(device=DEV)
    g.manual_seed(77)
    dO = torch.randn(B * T, H, d, device=DEV, generator=g).mul_(0.5).to(torch.bfloat16)
    cu_host = [i * T for i in range(B + 1)]
    _, st = gdn.gdn_cpr_forward(q, k, v, alpha, beta, cu, C, cu_seqlens_host=cu_host, out_dtype=torch.float32)
    grads = gdn.gdn_cpr_backward(q, k, v, alpha, beta, dO, st, cu, C, cu_seqlens_host=cu_host)
    torch.cuda.synchronize()
    n, h = 1, 29
    sl = slice(n * T, (n + 1) * T)
    host = lambda x: x[sl, h:h + 1].float().cpu().numpy()
    ref = oracle.adjoint(host(q), host(k), host(v), host(alpha), host(beta), host(dO),
                         np.array([0, T], np.int32), C)
    got = [x[sl, h:h + 1].cpu().numpy() for x in grads[:5]] + [grads[5][n:n + 1, h:h + 1].cpu().numpy()]
    check(got, ref, "trainer sample")


def test_backward_gate_extremes_vs_oracle():
    """alpha = 0 (a reset), alpha = 1, beta = 0 (no write) and beta = 1 at
    scattered tokens, in fp32; the gradient formulas hold at these values."""
    C, d = 32, 64
    b = synth.make_batch(77, [3 * C + 7, C, 5], 2, d, d, "f32")
    rng = np.random.default_rng(8)
    T = b.q.shape[0]
    for arr, vals in ((b.alpha, (0.0, 1.0)), (b.beta, (0.0, 1.0))):
        for val in vals:
            idx = rng.choice(T, size=T // 8, replace=False)
            arr[idx, rng.integers(0, 2, size=idx.size)] = val
    S0 = (rng.standard_normal((3, 2, d, d)) * 0.2).astype(np.float32)
    dO = _dO(12, T, 2, d, "f32")
    got = run(b, C, S0, dO)
    ref = oracle.adjoint(b.q, b.k, b.v, b.alpha, b.beta, dO, b.cu_seqlens, C, S0)
    check(got, ref, "gate extremes")


def test_backward_final_state_gradient_vs_oracle():
    """dstate_out (the loss gradient for each sequence's final state) against
    the oracle; an empty sequence passes it straight to dstate_in."""
    C, d, H = 32, 64, 2
    lens = [2 * C + 5, 0, C]
    b = synth.make_batch(91, lens, H, d, d, "bf16")
    rng = np.random.default_rng(19)
    S0 = (rng.standard_normal((3, H, d, d)) * 0.2).astype(np.float32)
    W = (rng.standard_normal((3, H, d, d)) * 0.1).astype(np.float32)
    dO = _dO(13, b.q.shape[0], H, d, "bf16")
    dd = to_device(b)
    _, st = gdn.gdn_cpr_forward(dd["q"], dd["k"], dd["v"], dd["alpha"], dd["beta"], dd["cu_seqlens"], C,
                                cu_seqlens_host=dd["cu_host"], state_in=torch.from_numpy(S0).to(DEV),
                                out_dtype=torch.float32)
    g = gdn.gdn_cpr_backward(dd["q"], dd["k"], dd["v"], dd["alpha"], dd["beta"],
                             torch.from_numpy(dO).to(DEV).to(torch.bfloat16), st, dd["cu_seqlens"], C,
                             cu_seqlens_host=dd["cu_host"], dstate_out=torch.from_numpy(W).to(DEV))
    torch.cuda.synchronize()
    got = [x.cpu().numpy() for x in g]
    ref = oracle.adjoint(b.q, b.k, b.v, b.alpha, b.beta, dO, b.cu_seqlens, C, S0, dstate_out=W)
    check(got, ref, "dstate_out")
    assert np.array_equal(bits(got[5][1]), bits(W[1]))


def test_backward_split_at_chunk_boundary_equals_unsplit_bitwise():
    """A sequence split at a chunk boundary: the later part's backward first,
    its dstate_in as the earlier part's dstate_out.  Every gradient equals the
    unsplit backward bit for bit (the trainer's bf16 shape)."""
    C, d, H = 64, 128, 2
    L, s = 5 * C + 9, 3 * C
    b = synth.make_batch(93, [L], H, d, d, "bf16")
    dd = to_device(b)
    rng = np.random.default_rng(23)
    S0 = torch.from_numpy((rng.standard_normal((1, H, d, d)) * 0.2).astype(np.float32)).to(DEV)
    W = torch.from_numpy((rng.standard_normal((1, H, d, d)) * 0.1).astype(np.float32)).to(DEV)
    dO = torch.from_numpy(_dO(17, L, H, d, "bf16")).to(DEV).to(torch.bfloat16)
    x = {n: dd[n] for n in ("q", "k", "v", "alpha", "beta")}

    def fwd_bwd(sl, state_in, dstate_out):
        part = {n: t[sl].contiguous() for n, t in x.items()}
        n_tok = part["q"].shape[0]
        cu = torch.tensor([0, n_tok], dtype=torch.int32, device=DEV)
        _, st = gdn.gdn_cpr_forward(part["q"], part["k"], part["v"], part["alpha"], part["beta"], cu, C,
                                    cu_seqlens_host=[0, n_tok], state_in=state_in)
        g = gdn.gdn_cpr_backward(part["q"], part["k"], part["v"], part["alpha"], part["beta"], dO[sl].contiguous(),
                                 st, cu, C, cu_seqlens_host=[0, n_tok], dstate_out=dstate_out)
        return st, g

    st_full, g_full = fwd_bwd(slice(0, L), S0, W)
    st1, _ = fwd_bwd(slice(0, s), S0, None)                 # the earlier part's forward: its last state
    _, g2 = fwd_bwd(slice(s, L), st1[-1:].contiguous(), W)  # the later part, from that state
    _, g1 = fwd_bwd(slice(0, s), S0, g2[5])                 # the earlier part, with the later part's dstate_in
    torch.cuda.synchronize()
    for i in range(5):
        assert np.array_equal(bits(g1[i]), bits(g_full[i][:s])), i
        assert np.array_equal(bits(g2[i]), bits(g_full[i][s:])), i
    assert np.array_equal(bits(g1[5]), bits(g_full[5]))
