"""Full-size workloads on the GPU, in the launch configuration the benchmark
times, checked on sampled (sequence, head) pairs the CPU oracle can compute,
plus GPU-vs-GPU bit identity over every output.

Inputs come from the device recipe of gated_deltanet_cpr_delta_b200.synth;
each sampled pair's inputs are copied to the host for the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import bits
from gated_deltanet_cpr_delta_b200 import gdn, synth

pytestmark = pytest.mark.gpu


def host_pair(d, n, h):
    """Inputs of sequence n, head h as fp32 numpy arrays [L,1,.] (exact values)."""
    a0, a1 = d["cu_host"][n], d["cu_host"][n + 1]
    g = lambda t: t[a0:a1, h:h + 1].float().cpu().numpy()
    return g(d["q"]), g(d["k"]), g(d["v"]), g(d["alpha"]), g(d["beta"]), np.array([0, a1 - a0], np.int32)


def check_pair(d, o, st, n, h, C, state_base, bf16_out=True):
    q, k, v, a, b, cu = host_pair(d, n, h)
    r = oracle.recurrent(q, k, v, a, b, cu, C)
    a0, a1 = d["cu_host"][n], d["cu_host"][n + 1]
    ns = (a1 - a0) // C + 1
    got_o = o[a0:a1, h:h + 1].float().cpu().numpy().astype(np.float64)
    got_s = st[state_base:state_base + ns, h:h + 1].cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got_o - r["o"])) <= 2e-2 * np.max(np.abs(r["o"]))
    assert np.max(np.abs(got_s - r["states"])) <= 2e-2 * np.max(np.abs(r["states"]))
    # per-token schedule bit-exact against the fp32 model, started from the GPU's boundary states
    mo, _, _ = oracle.schedule_tok_from_states(q, k, v, a, b, st[state_base:state_base + ns, h:h + 1].cpu().numpy(),
                                            cu, C)
    if bf16_out:
        assert np.array_equal(bits(o[a0:a1, h:h + 1].contiguous()), oracle.to_bf16_bits(mo))
    else:
        assert np.array_equal(bits(o[a0:a1, h:h + 1].contiguous()), bits(mo))


def test_prefill_workload_sampled():
    cfg = synth.PREFILL
    B, T, H, D, C = cfg["B"], cfg["T"], cfg["H"], cfg["dk"], cfg["C"]
    d = synth.make_batch_device(cfg["seed"], [T] * B, H, D, D, "bf16")
    o, st = gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"], C,
                                cu_seqlens_host=d["cu_host"])
    torch.cuda.synchronize()
    for n, h in [(0, 0), (3, 15), (1, 7)]:
        check_pair(d, o, st, n, h, C, n * (T // C + 1))
    # trainer forward is the same call: identical bits on a second invocation
    o2, st2 = gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"], C,
                                  cu_seqlens_host=d["cu_host"])
    assert torch.equal(o2.view(torch.int16), o.view(torch.int16))
    assert torch.equal(st2.view(torch.int32), st.view(torch.int32))


def test_decode_workload_prefill_then_decode_equals_full_prefill():
    cfg = synth.DECODE
    N, H, D, C = cfg["B"], cfg["H"], cfg["dk"], cfg["C"]
    Lp, steps = cfg["T_prefill"], cfg["steps"]
    L = Lp + steps
    d = synth.make_batch_device(cfg["seed"], [L] * N, H, D, D, "bf16")
    full_o, full_st = gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"], C,
                                          cu_seqlens_host=d["cu_host"])
    # prefill the first Lp tokens of every sequence, keeping a decode cache
    idx = torch.cat([torch.arange(n * L, n * L + Lp) for n in range(N)]).cuda()
    cu_p = [n * Lp for n in range(N + 1)]
    cache = gdn.new_cache(N, H, D, D, C, torch.bfloat16)
    gdn.gdn_cpr_forward(d["q"][idx], d["k"][idx], d["v"][idx], d["alpha"][idx], d["beta"][idx],
                        torch.tensor(cu_p, dtype=torch.int32, device="cuda"), C, cu_seqlens_host=cu_p,
                        cache_out=cache)
    outs = []
    for s in range(steps):
        t = torch.arange(N, device="cuda") * L + Lp + s
        outs.append(gdn.gdn_decode_step(d["q"][t], d["k"][t], d["v"][t], d["alpha"][t], d["beta"][t], cache, C))
    torch.cuda.synchronize()
    dec = torch.stack(outs, 1)                                   # [N, steps, H, D]
    ref = full_o.view(N, L, H, D)[:, Lp:]
    assert torch.equal(dec.view(torch.int16), ref.view(torch.int16))
    last = torch.arange(N, device="cuda") * (L // C + 1) + L // C
    assert torch.equal(cache["S_b"].view(torch.int32), full_st[last].view(torch.int32))
    assert torch.equal(cache["R"].view(torch.int32), full_st[last].view(torch.int32))  # L % C == 0
    assert int(cache["pos"].abs().max()) == 0
    for n, h in [(0, 0), (63, 31)]:
        check_pair(d, full_o, full_st, n, h, C, n * (L // C + 1))


def test_varlen_workload_batch_invariance():
    cfg = synth.VARLEN
    lens = synth.varlen_lengths(cfg["seed"], cfg["N"], cfg["lo"], cfg["hi"])
    H, D, C = cfg["H"], cfg["dk"], cfg["C"]
    d = synth.make_batch_device(cfg["seed"], lens, H, D, D, "bf16")
    o, st = gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"], C,
                                cu_seqlens_host=d["cu_host"])
    torch.cuda.synchronize()
    starts = np.concatenate([[0], np.cumsum([L // C + 1 for L in lens])])
    # each sequence alone, and at another batch position, gives the same bits
    for n in (int(np.argmax(lens)), 5, 31):
        a0, a1 = d["cu_host"][n], d["cu_host"][n + 1]
        for order in ([n], [n, 0] if n != 0 else [n, 1]):
            sl = torch.cat([torch.arange(d["cu_host"][m], d["cu_host"][m + 1]) for m in order[::-1]]).cuda()
            cu2 = [0]
            for m in order[::-1]:
                cu2.append(cu2[-1] + lens[m])
            o2, st2 = gdn.gdn_cpr_forward(d["q"][sl], d["k"][sl], d["v"][sl], d["alpha"][sl], d["beta"][sl],
                                          torch.tensor(cu2, dtype=torch.int32, device="cuda"), C,
                                          cu_seqlens_host=cu2)
            j = len(order) - 1                                   # n is last in the packed order
            b0 = cu2[j]
            sb = sum(lens[m] // C + 1 for m in order[::-1][:j])
            assert torch.equal(o2[b0:b0 + lens[n]].view(torch.int16), o[a0:a1].view(torch.int16))
            assert torch.equal(st2[sb:sb + lens[n] // C + 1].view(torch.int32),
                               st[starts[n]:starts[n + 1]].view(torch.int32))
    check_pair(d, o, st, int(np.argmax(lens)), 3, C, int(starts[int(np.argmax(lens))]))


def test_trainer_workload_sampled():
    cfg = synth.TRAIN
    B, T, H, D, C = cfg["B"], cfg["T"], cfg["H"], cfg["dk"], cfg["C"]
    d = synth.make_batch_device(cfg["seed"], [T] * B, H, D, D, "bf16")
    o, st = gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"], C,
                                cu_seqlens_host=d["cu_host"])
    torch.cuda.synchronize()
    check_pair(d, o, st, 1, 30, C, 1 * (T // C + 1))
