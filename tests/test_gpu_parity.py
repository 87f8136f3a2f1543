"""GPU parity of the CUDA path through the C ABI (small and ragged shapes).

* Bitwise against the fp32 schedule model (oracle/schedule_fp32.c) for the
  per-token schedule: o in fp32 and bf16 and the running cache state, with the
  model's P_tok started from the GPU's boundary states.  Those boundary states
  come from the tensor-core P_chunk; they are checked against the fp64 oracle
  within tolerance, and bit for bit across GPU paths.
* Within tolerance of the fp64 oracle: max|o - o*| <= 1e-4 for fp32 inputs,
  <= 2e-2 * ||o*||_inf for bf16 inputs; the same bounds for states.
* CPR self-consistency on the GPU, bit for bit: prefill == decode, split at a
  chunk boundary == unsplit, batch composition/packing invariance, repeats.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import bits, to_device
from gated_deltanet_cpr_delta_b200 import gdn, synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


def fwd(b, C, out_dtype=torch.float32, state_in=None, cache=False):
    d = to_device(b)
    c = None
    if cache:
        c = gdn.new_cache(len(d["cu_host"]) - 1, b.H, b.dk, b.dv, C, d["q"].dtype, DEV)
        c["pos"].fill_(-7)  # must be overwritten
    o, st = gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"], C,
                                cu_seqlens_host=d["cu_host"], state_in=state_in, out_dtype=out_dtype,
                                cache_out=c)
    torch.cuda.synchronize()
    return o, st, c


def tol_check(dtype, got, ref, what):
    err = np.max(np.abs(got.astype(np.float64) - ref)) if ref.size else 0.0
    if dtype == "f32":
        assert err <= 1e-4, (what, err)
    else:
        assert err <= 2e-2 * max(np.max(np.abs(ref)), 1e-30), (what, err)


# ------------------------------------------------------------------ tiny workload
def test_tiny_workload_bitwise_prefill_vs_decode_and_oracle():
    cfg = synth.TINY
    b = synth.make_batch(cfg["seed"], [cfg["T"]] * cfg["B"], cfg["H"], cfg["dk"], cfg["dv"], cfg["dtype"])
    C = cfg["C"]
    o, st, _ = fwd(b, C)
    mo, _, _ = oracle.schedule_tok_from_states(b.q, b.k, b.v, b.alpha, b.beta, st.cpu().numpy(), b.cu_seqlens, C)
    assert np.array_equal(bits(o), bits(mo))
    r = oracle.recurrent(b.q, b.k, b.v, b.alpha, b.beta, b.cu_seqlens, C)
    tol_check("f32", o.cpu().numpy(), r["o"], "o")
    tol_check("f32", st.cpu().numpy(), r["states"], "states")
    # the same 64 tokens through 64 decode steps, from a zero cache
    d = to_device(b)
    cache = gdn.new_cache(1, b.H, b.dk, b.dv, C, torch.float32, DEV)
    outs = [gdn.gdn_decode_step(d["q"][t:t + 1], d["k"][t:t + 1], d["v"][t:t + 1], d["alpha"][t:t + 1],
                                d["beta"][t:t + 1], cache, C) for t in range(cfg["T"])]
    torch.cuda.synchronize()
    assert np.array_equal(bits(torch.cat(outs)), bits(o))
    assert np.array_equal(bits(cache["S_b"][0]), bits(st[-1]))
    assert np.array_equal(bits(cache["R"][0]), bits(st[-1]))
    assert torch.all(cache["rscale"] == 1.0)
    assert int(cache["pos"].max()) == 0


# ------------------------------------------------------------------ all compiled shapes
SHAPES = [(d, C) for d in (16, 32, 64, 128) for C in (16, 32, 64)]


@pytest.mark.parametrize("d,C", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_forward_vs_schedule_model_and_oracle(d, C, dtype):
    lens = [1, C - 1, C, 0, C + 1, 3 * C + 5] if d <= 64 else [C - 1, 2 * C + 3, 0, C]
    H = 3 if d <= 64 else 2
    b = synth.make_batch(100 + d + C, lens, H, d, d, dtype)
    rng = np.random.default_rng(d * C)
    S0 = (rng.standard_normal((len(lens), H, d, d)) * 0.2).astype(np.float32)
    o, st, cache = fwd(b, C, torch.float32, torch.from_numpy(S0).to(DEV), cache=True)
    st_h = st.cpu().numpy()
    # P_tok bit for bit: the model's per-token schedule, started from the GPU's boundary states
    mo, mR, mRs = oracle.schedule_tok_from_states(b.q, b.k, b.v, b.alpha, b.beta, st_h, b.cu_seqlens, C)
    assert np.array_equal(bits(o), bits(mo))
    assert np.array_equal(bits(cache["R"]), bits(mR))
    assert np.array_equal(bits(cache["rscale"]), bits(mRs))
    # the first state of every sequence is state_in itself; S_b is the last boundary state
    first = np.concatenate([[0], np.cumsum([L // C + 1 for L in lens])])
    last = first[1:] - 1
    assert np.array_equal(bits(st_h[first[:-1]]), bits(S0))
    assert np.array_equal(bits(cache["S_b"]), bits(st_h[last]))
    m = oracle.schedule_forward(b.q, b.k, b.v, b.alpha, b.beta, b.cu_seqlens, C, S0, with_cache=True)
    pos = cache["pos"].cpu().numpy()
    assert np.array_equal(pos, m["pos"])
    for n in range(len(lens)):
        p = int(pos[n, 0])
        assert np.array_equal(cache["kbuf"][n, :, :p].float().cpu().numpy(), m["kbuf"][n, :, :p])
        assert np.array_equal(cache["vbuf"][n, :, :p].float().cpu().numpy(), m["vbuf"][n, :, :p])
        assert np.array_equal(cache["abuf"][n, :, :p].cpu().numpy(), m["abuf"][n, :, :p])
        assert np.array_equal(cache["bbuf"][n, :, :p].cpu().numpy(), m["bbuf"][n, :, :p])
    # bf16 output = nearest-even rounding of the same fp32 values
    o16, st16, _ = fwd(b, C, torch.bfloat16, torch.from_numpy(S0).to(DEV))
    assert np.array_equal(bits(o16), oracle.to_bf16_bits(mo))
    assert np.array_equal(bits(st16), bits(st))
    # fp64 oracle
    r = oracle.recurrent(b.q, b.k, b.v, b.alpha, b.beta, b.cu_seqlens, C, S0)
    tol_check(dtype, o.cpu().numpy(), r["o"], "o")
    tol_check(dtype, st.cpu().numpy(), r["states"], "states")


# 2C > d runs the resync as one kernel (k_dec_resync), 2C <= d as two (k_dec_rprep, k_dec_rstep)
@pytest.mark.parametrize("d,C,Lp,steps,dtype", [(16, 16, 0, 40, "bf16"), (16, 16, 21, 50, "bf16"),
                                                (64, 32, 64, 70, "bf16"), (128, 64, 130, 140, "bf16"),
                                                (128, 16, 16, 40, "bf16"), (64, 64, 70, 140, "bf16"),
                                                (64, 64, 70, 140, "f32"), (32, 32, 10, 80, "f32"),
                                                (128, 64, 60, 80, "f32")])
def test_decode_equals_prefill_bitwise(d, C, Lp, steps, dtype):
    N, H = 3, 2
    b = synth.make_batch(200 + d, [Lp + steps] * N, H, d, d, dtype)
    full_o, full_st, full_c = fwd(b, C, torch.float32, cache=True)
    cu = b.cu_seqlens
    if Lp > 0:
        sl = np.concatenate([np.arange(cu[n], cu[n] + Lp) for n in range(N)])
        pre = synth.Batch(b.q[sl], b.k[sl], b.v[sl], b.alpha[sl], b.beta[sl],
                          (np.arange(N + 1) * Lp).astype(np.int32), b.dtype)
        _, _, cache = fwd(pre, C, torch.float32, cache=True)
    else:
        cache = gdn.new_cache(N, H, d, d, C, torch.bfloat16 if dtype == "bf16" else torch.float32, DEV)
    dd = to_device(b)
    fo = full_o.cpu()
    for s in range(steps):
        idx = torch.from_numpy((cu[:-1] + Lp + s).astype(np.int64)).to(DEV)
        o = gdn.gdn_decode_step(dd["q"][idx], dd["k"][idx], dd["v"][idx], dd["alpha"][idx], dd["beta"][idx],
                                cache, C, out_dtype=torch.float32)
        assert np.array_equal(bits(o), bits(fo[idx.cpu()])), s
    torch.cuda.synchronize()
    for key in ("S_b", "R", "rscale", "pos"):
        assert np.array_equal(bits(cache[key]) if key != "pos" else cache[key].cpu().numpy(),
                              bits(full_c[key]) if key != "pos" else full_c[key].cpu().numpy()), key
    p = int(full_c["pos"][0, 0])
    for key in ("kbuf", "vbuf", "abuf", "bbuf"):
        assert torch.equal(cache[key][:, :, :p], full_c[key][:, :, :p]), key


def test_batch_composition_and_packing_invariance():
    C, d, H = 32, 64, 3
    lens = [200, 33, 64, 1, 97, 128]
    b = synth.make_batch(300, lens, H, d, d, "bf16")
    o, st, _ = fwd(b, C, torch.float32)
    starts = np.concatenate([[0], np.cumsum([L // C + 1 for L in lens])])
    perms = [[3, 0, 5], [5, 4, 3, 2, 1, 0], [1]]
    for perm in perms:
        pb = b.subset(perm)
        po, pst, _ = fwd(pb, C, torch.float32)
        pstarts = np.concatenate([[0], np.cumsum([lens[i] // C + 1 for i in perm])])
        for j, i in enumerate(perm):
            a0, a1 = b.cu_seqlens[i], b.cu_seqlens[i + 1]
            p0, p1 = pb.cu_seqlens[j], pb.cu_seqlens[j + 1]
            assert np.array_equal(bits(po[p0:p1]), bits(o[a0:a1]))
            assert np.array_equal(bits(pst[pstarts[j]:pstarts[j + 1]]), bits(st[starts[i]:starts[i + 1]]))
    # head subset: the same sequences with fewer heads
    hb = b.subset(range(len(lens)), heads=[2, 0])
    ho, _, _ = fwd(hb, C, torch.float32)
    assert np.array_equal(bits(ho), bits(o[:, [2, 0]].contiguous()))


def test_fused_chain_tok_path_equals_separate_kernels():
    """With d_v = 128 and fewer (sequence, head) pairs than SMs the library runs
    the boundary chain and P_tok as one cooperative kernel; with more pairs it
    runs them as separate kernels.  The same sequences give the same bits
    either way (ragged lengths, a partial last chunk, the decode cache)."""
    C, d, H = 64, 128, 4
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    lens = [300, 64, 1, 129, 0, 191]                       # 24 pairs: the fused kernel
    n_more = (sms + 64) // H                                # enough pairs for the separate kernels
    more = lens + [37 + 11 * i for i in range(n_more)]
    b = synth.make_batch(350, more, H, d, d, "bf16")
    o_big, st_big, c_big = fwd(b, C, torch.bfloat16, cache=True)
    small = b.subset(range(len(lens)))
    o, st, c = fwd(small, C, torch.bfloat16, cache=True)
    T = int(small.cu_seqlens[-1])
    ns = sum(L // C + 1 for L in lens)
    assert np.array_equal(bits(o), bits(o_big[:T]))
    assert np.array_equal(bits(st), bits(st_big[:ns]))
    for key in ("S_b", "R", "rscale", "pos"):
        assert torch.equal(c[key], c_big[key][:len(lens)]), key
    # and the fused result is the model's P_tok from the GPU's states, bit for bit
    mo, _, _ = oracle.schedule_tok_from_states(small.q, small.k, small.v, small.alpha, small.beta, st.cpu().numpy(),
                                            small.cu_seqlens, C)
    assert np.array_equal(bits(o), oracle.to_bf16_bits(mo))


def test_forward_and_decode_replay_from_cuda_graphs():
    """Both calls enqueue only stream work, so they can be captured into CUDA
    graphs (the fused cooperative kernel included); a replay gives the same
    bits as the eager calls."""
    C, d, H, N, L0, steps = 64, 128, 2, 3, 62, 4   # the decode steps cross a chunk boundary (a resync)
    b = synth.make_batch(360, [L0 + steps] * N, H, d, d, "bf16")
    dev = to_device(b)
    idx = torch.cat([torch.arange(n * (L0 + steps), n * (L0 + steps) + L0) for n in range(N)]).to(DEV)
    pre = {n: dev[n][idx].contiguous() for n in ("q", "k", "v", "alpha", "beta")}
    cu = [n * L0 for n in range(N + 1)]
    cu_dev = torch.tensor(cu, dtype=torch.int32, device=DEV)
    ws = torch.empty(gdn.gdn_cpr_workspace_size(N * L0, N, H, d, d, C), dtype=torch.uint8, device=DEV)
    o_e = torch.empty(N * L0, H, d, dtype=torch.bfloat16, device=DEV)
    st_e = torch.empty(gdn.gdn_num_chunk_states(cu, C), H, d, d, dtype=torch.float32, device=DEV)
    cache = gdn.new_cache(N, H, d, d, C, torch.bfloat16, DEV)
    fwd = lambda o, st, c: gdn.gdn_cpr_forward(pre["q"], pre["k"], pre["v"], pre["alpha"], pre["beta"], cu_dev, C,
                                               cu_seqlens_host=cu, o=o, chunk_states=st, workspace=ws, cache_out=c)
    fwd(o_e, st_e, cache)
    torch.cuda.synchronize()
    o_g, st_g = torch.zeros_like(o_e), torch.zeros_like(st_e)
    cache_g = {n: torch.zeros_like(t) for n, t in cache.items()}
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd(o_g, st_g, cache_g)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o_g.view(torch.int16), o_e.view(torch.int16)) and torch.equal(st_g, st_e)
    for n in cache:
        assert torch.equal(cache_g[n], cache[n]), n
    # decode: eager steps on one copy of the cache, graph replay on another
    step_in = []
    for s in range(steps):
        t = torch.arange(N, device=DEV) * (L0 + steps) + L0 + s
        step_in.append([dev[n][t].contiguous() for n in ("q", "k", "v", "alpha", "beta")])
    c_e = {n: t.clone() for n, t in cache.items()}
    outs_e = [gdn.gdn_decode_step(*step_in[s], c_e, C) for s in range(steps)]
    c_g = {n: t.clone() for n, t in cache.items()}
    outs_g = [torch.empty_like(outs_e[0]) for _ in range(steps)]
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2):
        for s in range(steps):
            gdn.gdn_decode_step(*step_in[s], c_g, C, o=outs_g[s])
    g2.replay()
    torch.cuda.synchronize()
    for s in range(steps):
        assert torch.equal(outs_g[s].view(torch.int16), outs_e[s].view(torch.int16)), s
    for n in c_e:
        assert torch.equal(c_g[n], c_e[n]), n


def test_split_at_chunk_boundary_equals_unsplit():
    C, d, H, L = 16, 32, 2, 150
    b = synth.make_batch(400, [L], H, d, d, "bf16")
    o, st, _ = fwd(b, C, torch.float32)
    for a in (16, 64, 144):
        p1 = synth.Batch(b.q[:a], b.k[:a], b.v[:a], b.alpha[:a], b.beta[:a], np.array([0, a], np.int32), "bf16")
        p2 = synth.Batch(b.q[a:], b.k[a:], b.v[a:], b.alpha[a:], b.beta[a:], np.array([0, L - a], np.int32),
                         "bf16")
        o1, s1, _ = fwd(p1, C, torch.float32)
        o2, s2, _ = fwd(p2, C, torch.float32, state_in=s1[-1:].contiguous())
        assert np.array_equal(bits(torch.cat([o1, o2])), bits(o))
        assert np.array_equal(bits(torch.cat([s1, s2[1:]])), bits(st))


def test_repeats_are_identical():
    C = 64
    b = synth.make_batch(500, [300, 129, 64], 4, 128, 128, "bf16")
    o0, s0, _ = fwd(b, C, torch.float32)
    for _ in range(10):
        o, s, _ = fwd(b, C, torch.float32)
        assert torch.equal(o.view(torch.int32), o0.view(torch.int32))
        assert torch.equal(s.view(torch.int32), s0.view(torch.int32))


def test_zero_length_and_empty_batches():
    C, d, H = 16, 16, 2
    b = synth.make_batch(600, [0, 0, 5], H, d, d, "f32")
    S0 = torch.randn(3, H, d, d, device=DEV)
    o, st, cache = fwd(b, C, torch.float32, S0, cache=True)
    assert st.shape[0] == 3
    assert torch.equal(st[0], S0[0]) and torch.equal(st[1], S0[1]) and torch.equal(st[2], S0[2])
    assert torch.equal(cache["S_b"][:2], S0[:2]) and torch.equal(cache["R"][:2], S0[:2])
    assert cache["pos"].cpu().tolist() == [[0, 0], [0, 0], [5, 5]]


def test_device_and_host_cu_seqlens_mismatch_writes_nothing():
    """The kernels check the device cu_seqlens against the host-derived totals
    and exit without writing when they disagree (outputs stay untouched)."""
    C, d, H = 16, 16, 2
    b = synth.make_batch(700, [40, 24], H, d, d, "f32")
    dd = to_device(b)
    bad_dev = torch.tensor([0, 24, 64], dtype=torch.int32, device=DEV)   # host says [0, 40, 64]
    o = torch.full((64, H, d), 7.0, device=DEV)
    st = torch.full((gdn.gdn_num_chunk_states(dd["cu_host"], C), H, d, d), 7.0, device=DEV)
    gdn.gdn_cpr_forward(dd["q"], dd["k"], dd["v"], dd["alpha"], dd["beta"], bad_dev, C,
                        cu_seqlens_host=dd["cu_host"], o=o, chunk_states=st)
    torch.cuda.synchronize()
    assert torch.all(o == 7.0) and torch.all(st == 7.0)


def test_invalid_decode_position_is_not_written_through():
    C, d, H = 16, 16, 1
    cache = gdn.new_cache(2, H, d, d, C, torch.float32, DEV)
    cache["R"].normal_()
    R0 = cache["R"].clone()
    cache["pos"][0] = 99
    b = synth.make_batch(800, [2], H, d, d, "f32")
    dd = to_device(b)
    gdn.gdn_decode_step(dd["q"], dd["k"], dd["v"], dd["alpha"], dd["beta"], cache, C)
    torch.cuda.synchronize()
    assert torch.equal(cache["R"][0], R0[0]) and int(cache["pos"][0, 0]) == 99
    assert not torch.equal(cache["R"][1], R0[1]) and int(cache["pos"][1, 0]) == 1
