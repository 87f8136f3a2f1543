"""Thin Python binding of the C ABI in include/gdn_cpr.h.

Argument marshalling only.  Torch tensors become device pointers, the current
torch CUDA stream becomes the stream handle, and output buffers are allocated
with torch.  Every step of the CPR path runs in the library's CUDA kernels.
There is no fallback: if libgdn_cpr.so is missing, or no GPU is present, the
calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn_cpr.so")

GDN_F32, GDN_BF16 = 0, 1
GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_WORKSPACE = 0, 1, 2, 3, 4
GDN_ERR_TIMEOUT, GDN_ERR_DEVICE_INPUT = 5, 6
_STATUS = {0: "GDN_OK", 1: "GDN_ERR_INVALID_ARG", 2: "GDN_ERR_UNSUPPORTED", 3: "GDN_ERR_CUDA",
           4: "GDN_ERR_WORKSPACE", 5: "GDN_ERR_TIMEOUT", 6: "GDN_ERR_DEVICE_INPUT"}

#: exported symbols of include/gdn_cpr.h
SYMBOLS = ("gdn_contract_id", "gdn_status_string", "gdn_num_chunk_states", "gdn_cpr_workspace_size",
           "gdn_cpr_forward", "gdn_decode_step", "gdn_cpr_forward_timed", "gdn_decode_step_timed",
           "gdn_decode_step_ex",
           "gdn_cpr_forward_noalloc", "gdn_contract_text", "gdn_contract_identity", "gdn_sha256_hex",
           "gdn_cpr_backward_workspace_size", "gdn_cpr_backward", "gdn_cpr_backward_timed",
           "gdn_read_device_status", "gdn_test_fault_injection")

#: gdn_identity_kind_t
ID_SEMANTIC, ID_NUMERICAL_POLICY, ID_DEPLOYMENT = 0, 1, 2

#: size of the fixed device array behind gdn_cpr_forward_noalloc (GDN_NOALLOC_SCRATCH_BYTES)
NOALLOC_SCRATCH_BYTES = 64 << 20


class GdnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_STATUS.get(status, status)} ({status})")
        self.status = status


class CacheStruct(ctypes.Structure):
    _fields_ = [("S_b", ctypes.c_void_p), ("R", ctypes.c_void_p), ("rscale", ctypes.c_void_p),
                ("kbuf", ctypes.c_void_p), ("vbuf", ctypes.c_void_p), ("abuf", ctypes.c_void_p),
                ("bbuf", ctypes.c_void_p), ("pos", ctypes.c_void_p), ("status", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libgdn_cpr.so (built by ``python -m gated_deltanet_cpr_delta_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with python -m gated_deltanet_cpr_delta_b200.build")
    lib = ctypes.CDLL(path)
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.gdn_contract_id.restype = ctypes.c_char_p
    lib.gdn_contract_id.argtypes = []
    lib.gdn_contract_text.restype = i64
    lib.gdn_contract_text.argtypes = [ctypes.c_int, i32, i32, i32, ctypes.c_int, ctypes.c_int, ctypes.c_char_p, sz]
    lib.gdn_contract_identity.restype = ctypes.c_int
    lib.gdn_contract_identity.argtypes = [ctypes.c_int, i32, i32, i32, ctypes.c_int, ctypes.c_int, ctypes.c_char_p]
    lib.gdn_sha256_hex.restype = ctypes.c_int
    lib.gdn_sha256_hex.argtypes = [ctypes.c_void_p, sz, ctypes.c_char_p]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_status_string.argtypes = [ctypes.c_int]
    lib.gdn_num_chunk_states.restype = i64
    lib.gdn_num_chunk_states.argtypes = [P, i32, i32]
    lib.gdn_cpr_workspace_size.restype = sz
    lib.gdn_cpr_workspace_size.argtypes = [i64, i32, i32, i32, i32, i32]
    lib.gdn_cpr_forward.restype = ctypes.c_int
    lib.gdn_cpr_forward.argtypes = [P, P, P, P, P, P, P, P, i32, i64, i32, i32, i32, i32, ctypes.c_int,
                                    ctypes.c_int, P, P, ctypes.POINTER(CacheStruct), P, sz, P]
    lib.gdn_decode_step.restype = ctypes.c_int
    lib.gdn_decode_step.argtypes = [P, P, P, P, P, ctypes.POINTER(CacheStruct), i32, i32, i32, i32, i32,
                                    ctypes.c_int, ctypes.c_int, P, P]
    lib.gdn_cpr_forward_timed.restype = ctypes.c_int
    lib.gdn_cpr_forward_timed.argtypes = lib.gdn_cpr_forward.argtypes + [P]
    lib.gdn_decode_step_timed.restype = ctypes.c_int
    lib.gdn_decode_step_timed.argtypes = lib.gdn_decode_step.argtypes + [P]
    lib.gdn_decode_step_ex.restype = ctypes.c_int
    lib.gdn_decode_step_ex.argtypes = lib.gdn_decode_step.argtypes[:-1] + [i32, P, P]
    lib.gdn_cpr_forward_noalloc.restype = ctypes.c_int
    lib.gdn_cpr_forward_noalloc.argtypes = [P, P, P, P, P, P, P, P, i32, i64, i32, i32, i32, i32, ctypes.c_int,
                                            ctypes.c_int, P, P, ctypes.POINTER(CacheStruct), P]
    lib.gdn_cpr_backward_workspace_size.restype = sz
    lib.gdn_cpr_backward_workspace_size.argtypes = [i64, i32, i32, i32, i32, i32]
    lib.gdn_cpr_backward.restype = ctypes.c_int
    lib.gdn_cpr_backward.argtypes = [P, P, P, P, P, P, P, P, P, P, i32, i64, i32, i32, i32, i32, ctypes.c_int,
                                     P, P, P, P, P, P, P, sz, P]
    lib.gdn_cpr_backward_timed.restype = ctypes.c_int
    lib.gdn_cpr_backward_timed.argtypes = lib.gdn_cpr_backward.argtypes + [P]
    lib.gdn_read_device_status.restype = ctypes.c_int
    lib.gdn_read_device_status.argtypes = [P, P, P]
    lib.gdn_test_fault_injection.restype = ctypes.c_int
    lib.gdn_test_fault_injection.argtypes = [i32, i64]
    _lib = lib
    return lib


def _dt(t: torch.dtype) -> int:
    if t == torch.float32:
        return GDN_F32
    if t == torch.bfloat16:
        return GDN_BF16
    raise ValueError(f"unsupported dtype {t}")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _event_array(events, n: int):
    """torch.cuda.Event list -> C array of cudaEvent_t handles (events must
    have been recorded once so that the CUDA event exists)."""
    if len(events) != n:
        raise ValueError(f"need {n} events")
    handles = [e.cuda_event for e in events]
    if any(h == 0 for h in handles):
        raise ValueError("record each event once before passing it (creates the CUDA event)")
    return (ctypes.c_void_p * n)(*handles)


def _check(st: int, what: str):
    if st != 0:
        raise GdnError(st, what)


def gdn_contract_id() -> str:
    return load_library().gdn_contract_id().decode()


def gdn_contract_text(kind: int, d_k: int, d_v: int, C: int, in_dtype: int, out_dtype: int) -> str:
    lib = load_library()
    n = lib.gdn_contract_text(kind, d_k, d_v, C, in_dtype, out_dtype, None, 0)
    if n < 0:
        raise GdnError(1, "gdn_contract_text")
    buf = ctypes.create_string_buffer(n + 1)
    lib.gdn_contract_text(kind, d_k, d_v, C, in_dtype, out_dtype, buf, n + 1)
    return buf.value.decode()


def gdn_contract_identity(kind: int, d_k: int, d_v: int, C: int, in_dtype: int, out_dtype: int) -> str:
    out = ctypes.create_string_buffer(65)
    _check(load_library().gdn_contract_identity(kind, d_k, d_v, C, in_dtype, out_dtype, out), "gdn_contract_identity")
    return out.value.decode()


def gdn_sha256_hex(data: bytes) -> str:
    out = ctypes.create_string_buffer(65)
    buf = ctypes.create_string_buffer(bytes(data), len(data))
    _check(load_library().gdn_sha256_hex(buf, len(data), out), "gdn_sha256_hex")
    return out.value.decode()


def gdn_num_chunk_states(cu_seqlens_host: Sequence[int], C: int) -> int:
    arr = (ctypes.c_int32 * len(cu_seqlens_host))(*[int(x) for x in cu_seqlens_host])
    n = load_library().gdn_num_chunk_states(arr, len(cu_seqlens_host) - 1, C)
    if n < 0:
        raise GdnError(1, "gdn_num_chunk_states")
    return int(n)


def gdn_cpr_workspace_size(total_tokens: int, num_seqs: int, H: int, d_k: int, d_v: int, C: int) -> int:
    return int(load_library().gdn_cpr_workspace_size(total_tokens, num_seqs, H, d_k, d_v, C))


def new_cache(N: int, H: int, d_k: int, d_v: int, C: int, dtype: torch.dtype, device="cuda",
              state: Optional[torch.Tensor] = None) -> Dict[str, torch.Tensor]:
    """Allocate a decode cache (gdn_cache_t layout).  With ``state`` [N,H,d_v,d_k]
    it starts at a chunk boundary with that state, otherwise at zero.  The
    running state is ``rscale * R``.  ``status`` is the decode step's device
    status word (one int32, starts at GDN_OK).  ``pos_host`` is a host copy of
    each sequence's buffer position (CPU int32 [N]): :func:`gdn_decode_step`
    skips the resync launch on steps where no buffer can fill."""
    S = torch.zeros(N, H, d_v, d_k, dtype=torch.float32, device=device) if state is None else state.clone()
    return dict(S_b=S, R=S.clone(), rscale=torch.ones(N, H, dtype=torch.float32, device=device),
                kbuf=torch.zeros(N, H, C, d_k, dtype=dtype, device=device),
                vbuf=torch.zeros(N, H, C, d_v, dtype=dtype, device=device),
                abuf=torch.zeros(N, H, C, dtype=torch.float32, device=device),
                bbuf=torch.zeros(N, H, C, dtype=torch.float32, device=device),
                pos=torch.zeros(N, H, dtype=torch.int32, device=device),
                status=torch.zeros(1, dtype=torch.int32, device=device),
                pos_host=torch.zeros(N, dtype=torch.int32))


def _set_pos_host(cache: Dict[str, torch.Tensor], cu_seqlens_host, C: int):
    """After a prefill into ``cache``: each sequence's position is L mod C."""
    cu = [int(x) for x in cu_seqlens_host]
    cache["pos_host"] = torch.tensor([(cu[n + 1] - cu[n]) % C for n in range(len(cu) - 1)], dtype=torch.int32)


def _cache_struct(c: Dict[str, torch.Tensor]) -> CacheStruct:
    st = c.get("status")
    return CacheStruct(*[c[n].data_ptr() for n in ("S_b", "R", "rscale", "kbuf", "vbuf", "abuf", "bbuf", "pos")],
                       st.data_ptr() if st is not None else None)


def read_device_status(workspace: Optional[torch.Tensor] = None, device=None) -> int:
    """The device status word of the last forward / backward that used
    ``workspace`` (None: the no-allocation forward's fixed array), read after
    the current stream has run that call (this synchronises the stream)."""
    dev = workspace.device if workspace is not None else torch.device("cuda", torch.cuda.current_device())
    out = torch.empty(1, dtype=torch.int32, device=dev)
    _check(load_library().gdn_read_device_status(_ptr(workspace), _ptr(out), _stream(dev)),
           "gdn_read_device_status")
    return int(out.item())


def set_fault_injection(mode: int, wait_clocks: int = 1 << 31) -> None:
    """Failure-detection hook (process-wide; mode 0 = off): see
    gdn_test_fault_injection in include/gdn_cpr.h."""
    _check(load_library().gdn_test_fault_injection(mode, wait_clocks), "gdn_test_fault_injection")


def gdn_cpr_forward(q, k, v, alpha, beta, cu_seqlens, C: int, *, cu_seqlens_host=None, state_in=None,
                    out_dtype=None, cache_out: Optional[Dict[str, torch.Tensor]] = None, workspace=None,
                    o=None, chunk_states=None, events=None):
    """CPR forward (prefill / trainer forward).

    q, k [T,H,d_k], v [T,H,d_v] (bf16 or fp32); alpha, beta [T,H] fp32;
    cu_seqlens int32 device [N+1] (``cu_seqlens_host``: the same values on the
    host; read back with a sync when omitted); state_in [N,H,d_v,d_k] fp32 or None.
    Returns (o [T,H,d_v] in out_dtype (default: q.dtype), chunk_states).
    ``events``: optional 6 torch.cuda.Events, recorded around the kernels
    (calls gdn_cpr_forward_timed).
    """
    lib = load_library()
    T, H, dk = k.shape
    dv = v.shape[2]
    if cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.cpu().tolist()
    cu_h = (ctypes.c_int32 * len(cu_seqlens_host))(*[int(x) for x in cu_seqlens_host])
    N = len(cu_seqlens_host) - 1
    out_dtype = q.dtype if out_dtype is None else out_dtype
    dev = k.device
    if o is None:
        o = torch.empty(T, H, dv, dtype=out_dtype, device=dev)
    if chunk_states is None:
        ns = lib.gdn_num_chunk_states(cu_h, N, C)
        if ns < 0:
            raise GdnError(1, "gdn_num_chunk_states")
        chunk_states = torch.empty(ns, H, dv, dk, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(lib.gdn_cpr_workspace_size(T, N, H, dk, dv, C), dtype=torch.uint8, device=dev)
    cs = _cache_struct(cache_out) if cache_out is not None else None
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state_in),
            _ptr(cu_seqlens), cu_h, N, T, H, dk, dv, C, _dt(q.dtype), _dt(out_dtype),
            _ptr(o), _ptr(chunk_states), ctypes.byref(cs) if cs is not None else None,
            _ptr(workspace), workspace.numel(), _stream(dev))
    if events is None:
        st = lib.gdn_cpr_forward(*args)
    else:
        st = lib.gdn_cpr_forward_timed(*args, _event_array(events, 6))
    _check(st, "gdn_cpr_forward")
    if cache_out is not None:
        _set_pos_host(cache_out, cu_seqlens_host, C)
    return o, chunk_states


def gdn_cpr_backward_workspace_size(total_tokens: int, num_seqs: int, H: int, d_k: int, d_v: int, C: int) -> int:
    return int(load_library().gdn_cpr_backward_workspace_size(total_tokens, num_seqs, H, d_k, d_v, C))


def gdn_cpr_backward(q, k, v, alpha, beta, dO, chunk_states, cu_seqlens, C: int, *, cu_seqlens_host=None,
                     dstate_out=None, workspace=None, grads=None, events=None):
    """CPR backward: gradients of sum(dO * o) for the forward of the same inputs.

    q, k, v, alpha, beta, cu_seqlens: as given to :func:`gdn_cpr_forward`;
    dO [T,H,d_v] in q's dtype; chunk_states: that forward's chunk states;
    dstate_out [N,H,d_v,d_k] fp32 or None: the loss gradient for each
    sequence's final state (a later part's dstate_in, when a sequence is split).
    Returns (dq, dk, dv, dalpha, dbeta, dstate_in), all fp32.  ``grads``: an
    optional tuple of those six tensors to write into.  ``events``: optional
    4 torch.cuda.Events recorded around the kernels (gdn_cpr_backward_timed)."""
    lib = load_library()
    T, H, dk = k.shape
    dv = v.shape[2]
    if cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.cpu().tolist()
    cu_h = (ctypes.c_int32 * len(cu_seqlens_host))(*[int(x) for x in cu_seqlens_host])
    N = len(cu_seqlens_host) - 1
    dev = k.device
    if grads is None:
        f32 = dict(dtype=torch.float32, device=dev)
        grads = (torch.empty(T, H, dk, **f32), torch.empty(T, H, dk, **f32), torch.empty(T, H, dv, **f32),
                 torch.empty(T, H, **f32), torch.empty(T, H, **f32), torch.empty(N, H, dv, dk, **f32))
    if workspace is None:
        workspace = torch.empty(lib.gdn_cpr_backward_workspace_size(T, N, H, dk, dv, C), dtype=torch.uint8,
                                device=dev)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(dO), _ptr(chunk_states), _ptr(dstate_out),
            _ptr(cu_seqlens), cu_h, N, T, H, dk, dv, C, _dt(q.dtype),
            *[_ptr(g) for g in grads], _ptr(workspace), workspace.numel(), _stream(dev))
    if events is None:
        st = lib.gdn_cpr_backward(*args)
    else:
        st = lib.gdn_cpr_backward_timed(*args, _event_array(events, 4))
    _check(st, "gdn_cpr_backward")
    return grads


def gdn_decode_step(q, k, v, alpha, beta, cache: Dict[str, torch.Tensor], C: int, *, out_dtype=None, o=None,
                    events=None):
    """One decode token per sequence.  q,k [N,H,d_k], v [N,H,d_v]; alpha, beta [N,H].
    ``cache`` (from :func:`new_cache` or a forward's ``cache_out``) is updated in place.
    ``events``: optional 3 torch.cuda.Events around the two kernels.  With the
    cache's ``pos_host`` (kept by :func:`new_cache`, the forwards and this call)
    the resync launch is skipped on steps where no sequence's buffer fills
    (gdn_decode_step_ex's hint); without it the resync is always launched."""
    lib = load_library()
    N, H, dk = k.shape
    dv = v.shape[2]
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if o is None:
        o = torch.empty(N, H, dv, dtype=out_dtype, device=k.device)
    cs = _cache_struct(cache)
    ph = cache.get("pos_host")
    ph = ph.numpy() if ph is not None else None  # numpy view of the CPU tensor: cheap host arithmetic
    may_resync = 1 if ph is None else int((ph >= C - 1).any())
    st = lib.gdn_decode_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), ctypes.byref(cs), N, H, dk,
                                dv, C, _dt(q.dtype), _dt(out_dtype), _ptr(o), may_resync, _stream(k.device),
                                _event_array(events, 3) if events is not None else None)
    _check(st, "gdn_decode_step")
    if ph is not None:
        ph += 1
        ph[ph >= C] = 0
    return o


def gdn_cpr_forward_noalloc(q, k, v, alpha, beta, cu_seqlens, C: int, *, cu_seqlens_host=None, state_in=None,
                            out_dtype=None, cache_out: Optional[Dict[str, torch.Tensor]] = None, o=None,
                            chunk_states=None):
    """CPR forward whose workspace is the library's fixed device array (see
    gdn_cpr_forward_noalloc in include/gdn_cpr.h): for callers that cannot
    allocate device memory when they call.  Same arguments and results as
    :func:`gdn_cpr_forward` without ``workspace``; ``o`` and ``chunk_states``
    should be passed in by such callers (they are allocated here only when
    omitted).  Calls that overlap on the GPU race on the shared array."""
    lib = load_library()
    T, H, dk = k.shape
    dv = v.shape[2]
    if cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.cpu().tolist()
    cu_h = (ctypes.c_int32 * len(cu_seqlens_host))(*[int(x) for x in cu_seqlens_host])
    N = len(cu_seqlens_host) - 1
    out_dtype = q.dtype if out_dtype is None else out_dtype
    dev = k.device
    if o is None:
        o = torch.empty(T, H, dv, dtype=out_dtype, device=dev)
    if chunk_states is None:
        chunk_states = torch.empty(gdn_num_chunk_states(cu_seqlens_host, C), H, dv, dk, dtype=torch.float32,
                                   device=dev)
    cs = _cache_struct(cache_out) if cache_out is not None else None
    st = lib.gdn_cpr_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state_in),
                                     _ptr(cu_seqlens), cu_h, N, T, H, dk, dv, C, _dt(q.dtype), _dt(out_dtype),
                                     _ptr(o), _ptr(chunk_states), ctypes.byref(cs) if cs is not None else None,
                                     _stream(dev))
    _check(st, "gdn_cpr_forward_noalloc")
    if cache_out is not None:
        _set_pos_host(cache_out, cu_seqlens_host, C)
    return o, chunk_states
