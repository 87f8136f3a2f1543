"""Forward and decode at the gate values where the gated delta rule has closed
forms: alpha = 0 (the state is reset), alpha = 1 with beta = 0 (the state is
kept), beta = 1 (the value is written).  They are planted at scattered tokens,
on a chunk's first and last token and over one whole chunk, and run through

* the separate-kernel forward (d = 64: the chain and the intra-chunk kernel
  are two launches),
* the fused forward (d = 128 with few (sequence, head) pairs: one
  cooperative launch),
* decode steps that cross a resync, started from a prefill's cache.

o and every chunk state are compared with the fp64 oracle (max error 1e-4 for
fp32 inputs, 2e-2 * ||o||_inf for bf16); o is compared bit for bit with the
fp32 schedule model's per-token steps started from the GPU's boundary states;
decode must equal the prefill of the same tokens bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import bits, to_device
from gated_deltanet_cpr_delta_b200 import gdn, synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


def plant_extremes(b, C, seed):
    """Gate extremes at fixed and random tokens of every sequence and head."""
    rng = np.random.default_rng(seed)
    a, be = b.alpha, b.beta
    for n in range(len(b.cu_seqlens) - 1):
        s0, s1 = int(b.cu_seqlens[n]), int(b.cu_seqlens[n + 1])
        L = s1 - s0
        if L == 0:
            continue
        a[s0, :] = 0.0                               # first token of the first chunk
        if L > C:
            a[s0 + C - 1, :] = 0.0                   # last token of chunk 0
            a[s0 + C, :] = 0.0                       # first token of chunk 1
        if L >= 3 * C:
            a[s0 + 2 * C:s0 + 3 * C, :] = 0.0        # one whole chunk of resets
        picks = rng.integers(s0, s1, size=(max(1, L // 7), 3))
        for t, hsel, kind in picks:
            h = int(hsel) % b.H
            if kind % 4 == 0:
                a[t, h] = 0.0
            elif kind % 4 == 1:
                a[t, h], be[t, h] = 1.0, 0.0         # state kept
            elif kind % 4 == 2:
                be[t, h] = 1.0                       # write
            else:
                a[t, h], be[t, h] = 1.0, 1.0
    return b


def tol(dtype, got, ref, what):
    err = float(np.max(np.abs(got.astype(np.float64) - ref))) if ref.size else 0.0
    bound = 1e-4 if dtype == "f32" else 2e-2 * max(float(np.max(np.abs(ref))), 1e-30)
    assert err <= bound, (what, err, bound)


def forward(b, C, out_dtype=torch.float32, cache=False):
    d = to_device(b)
    c = gdn.new_cache(len(d["cu_host"]) - 1, b.H, b.dk, b.dv, C, d["q"].dtype, DEV) if cache else None
    o, st = gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"], C,
                                cu_seqlens_host=d["cu_host"], out_dtype=out_dtype, cache_out=c)
    torch.cuda.synchronize()
    return o, st, c


@pytest.mark.parametrize("d,C,dtype,lens", [
    (64, 64, "f32", [200, 64, 1, 191, 0, 257]),       # separate kernels
    (64, 16, "bf16", [100, 48, 17]),                  # separate kernels, short chunks
    (128, 64, "bf16", [300, 64, 129, 1, 200]),        # fused kernel (few pairs)
    (128, 64, "f32", [257, 192]),                     # fused kernel, fp32 inputs
])
def test_forward_at_gate_extremes(d, C, dtype, lens):
    H = 3 if d == 64 else 2
    b = plant_extremes(synth.make_batch(1000 + d + C, lens, H, d, d, dtype), C, d * C)
    o, st, cache = forward(b, C, cache=True)
    st_h = st.cpu().numpy()
    mo, mR, mRs = oracle.schedule_tok_from_states(b.q, b.k, b.v, b.alpha, b.beta, st_h, b.cu_seqlens, C)
    assert np.array_equal(bits(o), bits(mo))
    assert np.array_equal(bits(cache["R"]), bits(mR))
    assert np.array_equal(bits(cache["rscale"]), bits(mRs))
    r = oracle.recurrent(b.q, b.k, b.v, b.alpha, b.beta, b.cu_seqlens, C)
    tol(dtype, o.cpu().numpy(), r["o"], "o")
    tol(dtype, st_h, r["states"], "states")
    # a whole chunk of resets: the state after it is exactly beta_t v_t k_t^T of
    # its last token (alpha = 0 removes everything before), so it is finite and small
    assert np.all(np.isfinite(st_h))


@pytest.mark.parametrize("d,C,Lp,steps", [(64, 16, 20, 45), (128, 64, 60, 140)])
def test_decode_across_resyncs_at_gate_extremes(d, C, Lp, steps):
    N, H = 3, 2
    b = plant_extremes(synth.make_batch(1100 + d, [Lp + steps] * N, H, d, d, "bf16"), C, 7 + d)
    # extra resets on the tokens the decode steps take at a chunk's edges
    for n in range(N):
        s0 = int(b.cu_seqlens[n])
        for t in range(Lp, Lp + steps):
            if t % C in (0, C - 1) and (t // C) % 2 == n % 2:
                b.alpha[s0 + t, :] = 0.0
    full_o, full_st, full_c = forward(b, C, cache=True)
    cu = b.cu_seqlens
    sl = np.concatenate([np.arange(cu[n], cu[n] + Lp) for n in range(N)])
    pre = synth.Batch(b.q[sl], b.k[sl], b.v[sl], b.alpha[sl], b.beta[sl], (np.arange(N + 1) * Lp).astype(np.int32),
                      b.dtype)
    _, _, cache = forward(pre, C, cache=True)
    dd = to_device(b)
    fo = full_o.cpu()
    for s in range(steps):
        idx = torch.from_numpy((cu[:-1] + Lp + s).astype(np.int64)).to(DEV)
        o = gdn.gdn_decode_step(dd["q"][idx], dd["k"][idx], dd["v"][idx], dd["alpha"][idx], dd["beta"][idx],
                                cache, C, out_dtype=torch.float32)
        assert np.array_equal(bits(o), bits(fo[idx.cpu()])), s
    torch.cuda.synchronize()
    for key in ("S_b", "R", "rscale", "pos"):
        assert torch.equal(cache[key], full_c[key]), key
    assert int(cache["status"].item()) == gdn.GDN_OK
    r = oracle.recurrent(b.q, b.k, b.v, b.alpha, b.beta, b.cu_seqlens, C)
    tol("bf16", full_o.cpu().numpy(), r["o"], "o")
    tol("bf16", full_st.cpu().numpy(), r["states"], "states")
