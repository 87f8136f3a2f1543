"""C-ABI checks that need no GPU: the library loads, exports every symbol
that include/gdn_cpr.h declares, sizes buffers, and rejects bad arguments on
the host before anything is enqueued."""
import ctypes
import os
import re

import pytest

from gated_deltanet_cpr_delta_b200 import build, gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return gdn.load_library()


def test_exports_every_declared_symbol(lib):
    hdr = open(os.path.join(ROOT, "include", "gdn_cpr.h")).read()
    declared = set(re.findall(r"^\S.*?\b(gdn_\w+)\s*\(", hdr, flags=re.M))
    assert declared == set(gdn.SYMBOLS)
    for s in declared:
        assert hasattr(lib, s), s


def test_contract_id(lib):
    assert gdn.gdn_contract_id() == "gdn-cpr-schedule-v6/NL8/ptok-scaled/prep-inverse-mma-tf32x3/chain-tcgen05-tf32x3-1acc"
    assert lib.gdn_status_string(0) == b"ok"
    assert lib.gdn_status_string(4) == b"workspace missing or too small"


def test_every_status_code_has_a_name(lib):
    hdr = open(os.path.join(ROOT, "include", "gdn_cpr.h")).read()
    codes = {int(v): n for n, v in re.findall(r"^\s*(GDN_(?:OK|ERR_\w+))\s*=\s*(\d+)", hdr, flags=re.M)}
    assert codes == {v: k for v, k in gdn._STATUS.items()}
    assert codes[5] == "GDN_ERR_TIMEOUT" and codes[6] == "GDN_ERR_DEVICE_INPUT"
    names = {c: lib.gdn_status_string(c) for c in codes}
    assert all(n != b"unknown status" for n in names.values())
    assert len(set(names.values())) == len(names)
    assert lib.gdn_status_string(99) == b"unknown status"


def test_fault_injection_and_status_read_validate_on_the_host(lib):
    # host-side argument checks only: nothing is enqueued, so no GPU is needed
    assert lib.gdn_test_fault_injection(2, 1000) == gdn.GDN_ERR_INVALID_ARG
    assert lib.gdn_test_fault_injection(1, 0) == gdn.GDN_ERR_INVALID_ARG
    assert lib.gdn_test_fault_injection(1, (1 << 31) + 1) == gdn.GDN_ERR_INVALID_ARG
    assert lib.gdn_test_fault_injection(0, 0) == gdn.GDN_OK
    assert lib.gdn_read_device_status(None, None, None) == gdn.GDN_ERR_INVALID_ARG


def test_num_chunk_states(lib):
    assert gdn.gdn_num_chunk_states([0, 64, 100, 100], 16) == 5 + 3 + 1
    assert gdn.gdn_num_chunk_states([0], 16) == 0
    with pytest.raises(gdn.GdnError):
        gdn.gdn_num_chunk_states([0, 10, 5], 16)        # decreasing
    with pytest.raises(gdn.GdnError):
        gdn.gdn_num_chunk_states([1, 10], 16)           # must start at 0


def test_workspace_size_grows_with_tokens(lib):
    a = gdn.gdn_cpr_workspace_size(1024, 2, 4, 64, 64, 16)
    b = gdn.gdn_cpr_workspace_size(2048, 2, 4, 64, 64, 16)
    assert 0 < a < b
    # w and u0 per full chunk and head dominate: C*(dk+dv) floats
    assert b - a >= (1024 // 16) * 4 * 16 * 128 * 4
    assert gdn.gdn_cpr_workspace_size(-1, 2, 4, 64, 64, 16) == 0


def _fwd(lib, **kw):
    P = ctypes.c_void_p
    cu = kw.get("cu", [0, 32])
    cu_h = (ctypes.c_int32 * len(cu))(*cu)
    fake = P(1 << 20)  # never dereferenced: validation fails first
    args = dict(q=fake, k=fake, v=fake, alpha=fake, beta=fake, state_in=None, cu=fake, cu_host=cu_h,
                N=len(cu) - 1, T=cu[-1], H=2, dk=16, dv=16, C=16, idt=0, odt=0, o=fake, states=fake,
                cache=None, ws=fake, wsb=1 << 30, stream=None)
    args.update({k: v for k, v in kw.items() if k != "cu"})
    return lib.gdn_cpr_forward(*args.values())


def test_forward_rejects_bad_arguments(lib):
    assert _fwd(lib, dk=24, dv=24) == 2                  # unsupported head dim
    assert _fwd(lib, dk=128, dv=64) == 2                 # d_k != d_v
    assert _fwd(lib, C=48) == 2                          # unsupported chunk
    assert _fwd(lib, idt=7) == 1                         # bad dtype
    assert _fwd(lib, cu=[0, 40, 32], T=32) == 1          # decreasing cu_seqlens
    assert _fwd(lib, cu=[0, 32], T=33) == 1              # total mismatch
    assert _fwd(lib, q=ctypes.c_void_p((1 << 20) + 4)) == 1   # misaligned
    assert _fwd(lib, states=None) == 1
    assert _fwd(lib, wsb=16) == 4                        # workspace too small
    assert _fwd(lib, ws=None) == 4
    assert _fwd(lib, H=0) == 1


def test_decode_rejects_bad_arguments(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)
    cs = gdn.CacheStruct(*([1 << 20] * 7))
    ok = dict(q=fake, k=fake, v=fake, a=fake, b=fake, cache=ctypes.byref(cs), N=2, H=2, dk=16, dv=16, C=16,
              idt=1, odt=1, o=fake, s=None)
    bad = dict(ok, C=8)
    assert lib.gdn_decode_step(*bad.values()) == 2
    bad = dict(ok, cache=None)
    assert lib.gdn_decode_step(*bad.values()) == 1
    bad = dict(ok, o=None)
    assert lib.gdn_decode_step(*bad.values()) == 1
    cs2 = gdn.CacheStruct(*([1 << 20] * 6 + [0]))
    bad = dict(ok, cache=ctypes.byref(cs2))
    assert lib.gdn_decode_step(*bad.values()) == 1


def _bwd(lib, **kw):
    P = ctypes.c_void_p
    cu = kw.get("cu", [0, 32])
    cu_h = (ctypes.c_int32 * len(cu))(*cu)
    fake = P(1 << 20)  # never dereferenced: validation fails first
    args = dict(q=fake, k=fake, v=fake, alpha=fake, beta=fake, dO=fake, states=fake, ds_out=None, cu=fake, cu_host=cu_h,
                N=len(cu) - 1, T=cu[-1], H=2, dk=16, dv=16, C=16, idt=0, dq=fake, dk_=fake, dv_=fake, da=fake,
                db=fake, ds=fake, ws=fake, wsb=1 << 30, stream=None)
    args.update({k: v for k, v in kw.items() if k != "cu"})
    return lib.gdn_cpr_backward(*args.values())


def test_backward_rejects_bad_arguments(lib):
    assert _bwd(lib, dk=24, dv=24) == 2                  # unsupported head dim
    assert _bwd(lib, C=48) == 2                          # unsupported chunk
    assert _bwd(lib, idt=7) == 1                         # bad dtype
    assert _bwd(lib, cu=[0, 40, 32], T=32) == 1          # decreasing cu_seqlens
    assert _bwd(lib, cu=[0, 32], T=33) == 1              # total mismatch
    assert _bwd(lib, dO=ctypes.c_void_p((1 << 20) + 4)) == 1   # misaligned
    assert _bwd(lib, states=None) == 1
    assert _bwd(lib, ds=None) == 1
    assert _bwd(lib, ds_out=ctypes.c_void_p((1 << 20) + 8)) == 1   # misaligned final-state gradient
    assert _bwd(lib, dq=None) == 1
    assert _bwd(lib, wsb=16) == 4                        # workspace too small
    assert _bwd(lib, ws=None) == 4
    assert _bwd(lib, H=0) == 1


def test_backward_workspace_size_grows_with_tokens():
    a = gdn.gdn_cpr_backward_workspace_size(1024, 2, 4, 128, 128, 64)
    b = gdn.gdn_cpr_backward_workspace_size(2048, 2, 4, 128, 128, 64)
    # at least the per-tile partial sums of dq and dk for the extra tokens
    assert b - a >= 1024 * 4 * 4 * 128 * 4 * 2
    assert gdn.gdn_cpr_backward_workspace_size(-1, 2, 4, 64, 64, 16) == 0
