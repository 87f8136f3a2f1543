"""Device-side error reporting through the C ABI.

Two errors can only be seen while the kernels run: a device cu_seqlens that
disagrees with the host copy, and a bounded wait that runs out.  The kernels
record them in a status word (the workspace's first word for the forward and
the backward, gdn_cache_t.status for decode), which gdn_read_device_status
copies out.  The timeout is made on purpose with the failure-detection hook:
the fused forward kernel withholds its boundary-state publications, so every
intra-chunk task waits for a state that never comes; each wait is bounded
(a few milliseconds here), records GDN_ERR_TIMEOUT and ends.  Nothing faults
or hangs, and the context stays usable (checked by a normal call afterwards).
"""
import numpy as np
import pytest
import torch

from conftest import bits, to_device
from gated_deltanet_cpr_delta_b200 import gdn, synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _fwd(d, C, ws, cu_dev=None, o=None, st=None):
    o, st = gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                                d["cu_seqlens"] if cu_dev is None else cu_dev, C, cu_seqlens_host=d["cu_host"],
                                out_dtype=torch.float32, workspace=ws, o=o, chunk_states=st)
    return o, st


def _ws(d, C):
    T, H, D = d["k"].shape
    return torch.empty(gdn.gdn_cpr_workspace_size(T, len(d["cu_host"]) - 1, H, D, D, C), dtype=torch.uint8,
                       device=DEV)


def test_forward_status_ok_then_device_input_then_ok():
    C, D, H = 16, 16, 2
    b = synth.make_batch(710, [40, 24], H, D, D, "f32")
    d = to_device(b)
    ws = _ws(d, C)
    o_ref, st_ref = _fwd(d, C, ws)
    assert gdn.read_device_status(ws) == gdn.GDN_OK
    bad = torch.tensor([0, 24, 64], dtype=torch.int32, device=DEV)   # the host copy says [0, 40, 64]
    o = torch.full_like(o_ref, 7.0)
    st = torch.full_like(st_ref, 7.0)
    _fwd(d, C, ws, cu_dev=bad, o=o, st=st)
    assert gdn.read_device_status(ws) == gdn.GDN_ERR_DEVICE_INPUT
    assert torch.all(o == 7.0) and torch.all(st == 7.0)
    # the next good call resets the word
    o2, st2 = _fwd(d, C, ws)
    assert gdn.read_device_status(ws) == gdn.GDN_OK
    assert torch.equal(o2, o_ref) and torch.equal(st2, st_ref)


def test_backward_status_reports_device_input():
    C, D, H = 16, 32, 2
    b = synth.make_batch(720, [50, 30], H, D, D, "bf16")
    d = to_device(b)
    o, st = gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"], C,
                                cu_seqlens_host=d["cu_host"])
    dO = torch.randn_like(o)
    T = int(b.cu_seqlens[-1])
    wsb = torch.empty(gdn.gdn_cpr_backward_workspace_size(T, 2, H, D, D, C), dtype=torch.uint8, device=DEV)
    gdn.gdn_cpr_backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], dO, st, d["cu_seqlens"], C,
                         cu_seqlens_host=d["cu_host"], workspace=wsb)
    assert gdn.read_device_status(wsb) == gdn.GDN_OK
    bad = torch.tensor([0, 30, 80], dtype=torch.int32, device=DEV)   # the host copy says [0, 50, 80]
    gdn.gdn_cpr_backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], dO, st, bad, C,
                         cu_seqlens_host=d["cu_host"], workspace=wsb)
    assert gdn.read_device_status(wsb) == gdn.GDN_ERR_DEVICE_INPUT


def test_bounded_wait_runs_out_and_reports_timeout():
    """Fused forward (d = 128, few pairs) with its boundary states withheld:
    every wait gives up after ~4M clocks and the call reports GDN_ERR_TIMEOUT."""
    C, D, H = 64, 128, 2
    b = synth.make_batch(730, [300, 129], H, D, D, "bf16")
    d = to_device(b)
    ws = _ws(d, C)
    o_ref, st_ref = _fwd(d, C, ws)
    torch.cuda.synchronize()
    assert gdn.read_device_status(ws) == gdn.GDN_OK
    o = torch.full_like(o_ref, 7.0)
    try:
        gdn.set_fault_injection(1, 1 << 22)
        _fwd(d, C, ws, o=o)
        torch.cuda.synchronize()
    finally:
        gdn.set_fault_injection(0)
    assert gdn.read_device_status(ws) == gdn.GDN_ERR_TIMEOUT
    assert torch.all(o == 7.0)  # no task passed its wait, so no output was written
    # the context is still usable, and a normal call gives the normal bits
    o2, st2 = _fwd(d, C, ws)
    assert gdn.read_device_status(ws) == gdn.GDN_OK
    assert np.array_equal(bits(o2), bits(o_ref)) and np.array_equal(bits(st2), bits(st_ref))


def test_decode_status_records_an_invalid_position():
    C, D, H = 16, 16, 1
    cache = gdn.new_cache(2, H, D, D, C, torch.float32, DEV)
    b = synth.make_batch(740, [2], H, D, D, "f32")
    d = to_device(b)
    gdn.gdn_decode_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"], cache, C)
    torch.cuda.synchronize()
    assert int(cache["status"].item()) == gdn.GDN_OK
    cache["pos"][0] = 99
    gdn.gdn_decode_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"], cache, C)
    torch.cuda.synchronize()
    assert int(cache["status"].item()) == gdn.GDN_ERR_DEVICE_INPUT
    assert int(cache["pos"][0, 0]) == 99 and int(cache["pos"][1, 0]) == 2


def test_decode_resync_hint_skips_the_launch_and_a_wrong_hint_is_reported():
    """The host hint (gdn_decode_step_ex, may_resync): the binding's pos_host
    skips the resync launch only where no buffer fills, and the results equal
    the always-resync path bit for bit across a boundary.  A wrong hint leaves
    the filled pair at pos = C; the next step refuses that position
    (GDN_ERR_DEVICE_INPUT, nothing written) and a resync brings it back."""
    C, D, H, N = 16, 16, 2, 2
    Lp, steps = 13, 6  # the 3rd step fills the buffers
    b = synth.make_batch(760, [Lp + steps] * N, H, D, D, "bf16")
    cu = b.cu_seqlens
    sl = np.concatenate([np.arange(cu[n], cu[n] + Lp) for n in range(N)])
    pre = synth.Batch(b.q[sl], b.k[sl], b.v[sl], b.alpha[sl], b.beta[sl], (np.arange(N + 1) * Lp).astype(np.int32),
                      b.dtype)
    dd = to_device(b)

    def prefill():
        d = to_device(pre)
        c = gdn.new_cache(N, H, D, D, C, d["q"].dtype, DEV)
        gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"], C,
                            cu_seqlens_host=d["cu_host"], out_dtype=torch.float32, cache_out=c)
        return c

    hinted, always = prefill(), prefill()
    assert hinted["pos_host"].tolist() == [Lp % C] * N
    del always["pos_host"]  # no host positions: every step launches the resync
    for s in range(steps):
        idx = torch.from_numpy((cu[:-1] + Lp + s).astype(np.int64)).to(DEV)
        args = (dd["q"][idx], dd["k"][idx], dd["v"][idx], dd["alpha"][idx], dd["beta"][idx])
        o1 = gdn.gdn_decode_step(*args, hinted, C, out_dtype=torch.float32)
        o2 = gdn.gdn_decode_step(*args, always, C, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert np.array_equal(bits(o1), bits(o2)), s
    for key in ("S_b", "R", "rscale", "pos", "kbuf", "vbuf"):
        assert torch.equal(hinted[key], always[key]), key
    assert hinted["pos_host"].tolist() == [(Lp + steps) % C] * N
    assert int(hinted["status"].item()) == gdn.GDN_OK

    # a wrong hint: the binding believes the step cannot fill a buffer
    wrong = prefill()
    for s in range(2):
        idx = torch.from_numpy((cu[:-1] + Lp + s).astype(np.int64)).to(DEV)
        gdn.gdn_decode_step(dd["q"][idx], dd["k"][idx], dd["v"][idx], dd["alpha"][idx], dd["beta"][idx], wrong, C)
    wrong["pos_host"][:] = 0
    idx = torch.from_numpy((cu[:-1] + Lp + 2).astype(np.int64)).to(DEV)
    step3 = (dd["q"][idx], dd["k"][idx], dd["v"][idx], dd["alpha"][idx], dd["beta"][idx])
    gdn.gdn_decode_step(*step3, wrong, C)
    torch.cuda.synchronize()
    assert (wrong["pos"] == C).all() and int(wrong["status"].item()) == gdn.GDN_OK
    del wrong["pos_host"]  # next step: unknown positions, the resync runs after the refused token
    gdn.gdn_decode_step(*step3, wrong, C)
    torch.cuda.synchronize()
    assert int(wrong["status"].item()) == gdn.GDN_ERR_DEVICE_INPUT
    assert torch.equal(wrong["S_b"], always["S_b"])  # the resync over the full buffer happened
    assert (wrong["pos"] == 0).all()
