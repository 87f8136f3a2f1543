"""The forward that allocates nothing (gdn_cpr_forward_noalloc).

Some callers cannot allocate device memory when they call the layer: a
plugin whose host framework owns all device memory and forbids allocation
inside its execute callback, or a process that has reserved the whole device
for its own pool.  For them the library keeps a fixed workspace array in its
own module.  This test calls that entry point directly through the C ABI and
checks, on two calls in a row, that its outputs match the regular
gdn_cpr_forward (caller-provided workspace) within the tolerance the other
parity tests use; the two paths run the same kernels, so the bits match.
It also checks that a batch too large for the fixed array is refused.

The file name sorts last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from conftest import bits, to_device
from gated_deltanet_cpr_delta_b200 import gdn, synth

pytestmark = pytest.mark.gpu


def _noalloc_raw(d, C, o, st, state_in=None):
    """Call gdn_cpr_forward_noalloc through the C ABI (ctypes)."""
    lib = gdn.load_library()
    T, H, dk = d["k"].shape
    dv = d["v"].shape[2]
    cu_h = (ctypes.c_int32 * len(d["cu_host"]))(*d["cu_host"])
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return lib.gdn_cpr_forward_noalloc(P(d["q"]), P(d["k"]), P(d["v"]), P(d["alpha"]), P(d["beta"]),
                                       P(state_in), P(d["cu_seqlens"]), cu_h, len(d["cu_host"]) - 1, T, H, dk, dv,
                                       C, gdn.GDN_BF16, gdn.GDN_F32, P(o), P(st), None,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_forward_matches_regular_forward_twice():
    C, D, H = 32, 64, 4
    # two different batches in a row: the second call must not see the first's leftovers
    for seed, lens in ((900, [100, 64, 33, 0, 129]), (901, [31, 250])):
        b = synth.make_batch(seed, lens, H, D, D, "bf16")
        d = to_device(b)
        S0 = torch.randn(len(lens), H, D, D, device="cuda") * 0.1
        o_ref, st_ref = gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"], C,
                                            cu_seqlens_host=d["cu_host"], state_in=S0, out_dtype=torch.float32)
        o = torch.full_like(o_ref, float("nan"))
        st = torch.full_like(st_ref, float("nan"))
        assert _noalloc_raw(d, C, o, st, S0) == 0
        torch.cuda.synchronize()
        ref_o, got_o = o_ref.double().cpu().numpy(), o.double().cpu().numpy()
        assert np.max(np.abs(got_o - ref_o)) <= 2e-2 * np.max(np.abs(ref_o))
        assert np.array_equal(bits(o), bits(o_ref))
        assert np.array_equal(bits(st), bits(st_ref))


def test_noalloc_forward_refuses_batches_beyond_the_fixed_array():
    C, D, H = 64, 128, 16
    T = 8192  # 128 chunks x 16 heads x 64 KiB of w/u0 > 64 MiB
    assert gdn.gdn_cpr_workspace_size(T, 1, H, D, D, C) > gdn.NOALLOC_SCRATCH_BYTES
    d = dict(q=torch.empty(T, H, D, dtype=torch.bfloat16, device="cuda"),
             k=torch.empty(T, H, D, dtype=torch.bfloat16, device="cuda"),
             v=torch.empty(T, H, D, dtype=torch.bfloat16, device="cuda"),
             alpha=torch.empty(T, H, device="cuda"), beta=torch.empty(T, H, device="cuda"),
             cu_seqlens=torch.tensor([0, T], dtype=torch.int32, device="cuda"), cu_host=[0, T])
    o = torch.empty(T, H, D, device="cuda")
    st = torch.empty(T // C + 1, H, D, D, device="cuda")
    assert _noalloc_raw(d, C, o, st) == 4  # GDN_ERR_WORKSPACE, nothing enqueued
