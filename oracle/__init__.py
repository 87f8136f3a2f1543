"""CPU oracle of the CPR Gated DeltaNet path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
``cpu_baseline`` / reference leg may import this package.  The product
library never loads it, and it shares no code with the CUDA path.

Contents
--------
* :func:`recurrent` -- fp64 token-by-token gated delta rule (C, OpenMP over
  (sequence, head)).  The plain definition the CPR evaluation must reach.
* :func:`chunkwise` -- an independent fp64 chunkwise form (numpy + a
  library triangular solve), see :mod:`oracle.chunkwise`.
* :mod:`oracle.exact` -- exact rational recurrence and exact binary32
  rounding, for tiny inputs.
* :func:`schedule_forward`, :func:`schedule_decode_step` -- scalar fp32
  model (C) of the written-down arithmetic schedule, the bit pattern the
  CUDA kernels must reproduce.
"""
from __future__ import annotations

import ctypes
import numpy as np

from . import build as _build
from . import chunkwise as _chunkwise
from . import chunkwise_adjoint as _chunkwise_adjoint

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32 = ctypes.c_int32
        lib.oracle_recurrent_fp64.restype = ctypes.c_int
        lib.oracle_recurrent_fp64.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, P, P, P]
        lib.oracle_adjoint_fp64.restype = ctypes.c_int
        lib.oracle_adjoint_fp64.argtypes = [P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, P, P, P, P, P, P]
        lib.sched_forward.restype = ctypes.c_int
        lib.sched_forward.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                      P, P, P, P, P, P, P, P, P, P]
        lib.sched_decode_step.restype = ctypes.c_int
        lib.sched_decode_step.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P,
                                          i32, i32, i32, i32, i32, P]
        lib.sched_f32_to_bf16.restype = None
        lib.sched_f32_to_bf16.argtypes = [P, P, ctypes.c_int64]
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return None if a is None else np.ascontiguousarray(a, dtype=dt)


def num_chunk_states(cu_seqlens, C):
    cu = np.asarray(cu_seqlens, np.int64)
    return int(sum(int(cu[i + 1] - cu[i]) // C + 1 for i in range(cu.shape[0] - 1)))


def recurrent(q, k, v, alpha, beta, cu_seqlens, C, state_in=None):
    """fp64 recurrence.  Arrays are widened exactly to float64.

    Returns dict(o [T,H,dv], states [sum(L//C+1),H,dv,dk], final [N,H,dv,dk]).
    """
    lib = _load()
    q, k, v = _c(q, np.float64), _c(k, np.float64), _c(v, np.float64)
    alpha, beta = _c(alpha, np.float64), _c(beta, np.float64)
    cu = _c(cu_seqlens, np.int32)
    T, H, dk = k.shape
    dv = v.shape[2]
    N = cu.shape[0] - 1
    s_in = _c(state_in, np.float64)
    o = np.zeros((T, H, dv))
    states = np.zeros((num_chunk_states(cu, C), H, dv, dk))
    final = np.zeros((N, H, dv, dk))
    rc = lib.oracle_recurrent_fp64(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(s_in), _p(cu),
                                   N, H, dk, dv, C, _p(o), _p(states), _p(final))
    if rc:
        raise RuntimeError(f"oracle_recurrent_fp64 failed ({rc})")
    return dict(o=o, states=states, final=final)


def adjoint(q, k, v, alpha, beta, dO, cu_seqlens, C, state_in=None, dstate_out=None):
    """fp64 gradient of L = sum_t dO_t . o_t (+ <dstate_out, final state> per
    sequence and head, when given) through the recurrence
    (oracle/adjoint_fp64.c).  Returns dict(dq, dk, dv, dalpha, dbeta,
    dstate_in [N,H,dv,dk])."""
    lib = _load()
    q, k, v = _c(q, np.float64), _c(k, np.float64), _c(v, np.float64)
    alpha, beta, dO = _c(alpha, np.float64), _c(beta, np.float64), _c(dO, np.float64)
    cu = _c(cu_seqlens, np.int32)
    T, H, dk = k.shape
    dv = v.shape[2]
    N = cu.shape[0] - 1
    s_in = _c(state_in, np.float64)
    s_out = _c(dstate_out, np.float64)
    out = dict(dq=np.zeros((T, H, dk)), dk=np.zeros((T, H, dk)), dv=np.zeros((T, H, dv)),
               dalpha=np.zeros((T, H)), dbeta=np.zeros((T, H)), dstate_in=np.zeros((N, H, dv, dk)))
    rc = lib.oracle_adjoint_fp64(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(s_in), _p(s_out), _p(dO), _p(cu), N, H, dk, dv, C,
                                 _p(out["dq"]), _p(out["dk"]), _p(out["dv"]), _p(out["dalpha"]), _p(out["dbeta"]),
                                 _p(out["dstate_in"]))
    if rc:
        raise RuntimeError(f"oracle_adjoint_fp64 failed ({rc})")
    return out


def adjoint_chunkwise(q, k, v, alpha, beta, dO, cu_seqlens, C, state_in=None, dstate_out=None,
                      dtype=np.float64):
    """Independent chunkwise form of the adjoint (see :mod:`oracle.chunkwise_adjoint`),
    fp64 unless ``dtype`` says otherwise."""
    return _chunkwise_adjoint.adjoint(q, k, v, alpha, beta, dO, cu_seqlens, C, state_in, dstate_out, dtype)


def chunkwise(q, k, v, alpha, beta, cu_seqlens, C, state_in=None):
    """Independent fp64 chunkwise form (see :mod:`oracle.chunkwise`)."""
    return _chunkwise.forward(q, k, v, alpha, beta, cu_seqlens, C, state_in)


def schedule_forward(q, k, v, alpha, beta, cu_seqlens, C, state_in=None, with_cache=False):
    """fp32 schedule model of the CPR forward.  Inputs must be fp32-valued
    (bf16 inputs widened exactly).  Returns dict(o (fp32, before the output
    cast), states, and with_cache: S_b, R, kbuf, vbuf, abuf, bbuf, pos, rscale),
    the running state being rscale * R."""
    lib = _load()
    q, k, v = _c(q, np.float32), _c(k, np.float32), _c(v, np.float32)
    alpha, beta = _c(alpha, np.float32), _c(beta, np.float32)
    cu = _c(cu_seqlens, np.int32)
    T, H, dk = k.shape
    dv = v.shape[2]
    N = cu.shape[0] - 1
    s_in = _c(state_in, np.float32)
    o = np.zeros((T, H, dv), np.float32)
    states = np.zeros((num_chunk_states(cu, C), H, dv, dk), np.float32)
    out = dict(o=o, states=states)
    cache = [None] * 8
    if with_cache:
        cache = [np.zeros((N, H, dv, dk), np.float32), np.zeros((N, H, dv, dk), np.float32),
                 np.zeros((N, H, C, dk), np.float32), np.zeros((N, H, C, dv), np.float32),
                 np.zeros((N, H, C), np.float32), np.zeros((N, H, C), np.float32),
                 np.zeros((N, H), np.int32), np.zeros((N, H), np.float32)]
        out.update(zip(["S_b", "R", "kbuf", "vbuf", "abuf", "bbuf", "pos", "rscale"], cache))
    rc = lib.sched_forward(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(s_in), _p(cu),
                           N, H, dk, dv, C, _p(o), _p(states), *[_p(a) for a in cache])
    if rc:
        raise RuntimeError(f"sched_forward failed ({rc})")
    return out


def schedule_decode_step(cache, q, k, v, alpha, beta, C):
    """One decode step of the fp32 schedule model; ``cache`` (dict from
    :func:`schedule_forward` with_cache=True) is updated in place.
    q,k [N,H,dk], v [N,H,dv], alpha/beta [N,H].  Returns o [N,H,dv] fp32."""
    lib = _load()
    q, k, v = _c(q, np.float32), _c(k, np.float32), _c(v, np.float32)
    alpha, beta = _c(alpha, np.float32), _c(beta, np.float32)
    N, H, dk = k.shape
    dv = v.shape[2]
    o = np.zeros((N, H, dv), np.float32)
    rc = lib.sched_decode_step(_p(q), _p(k), _p(v), _p(alpha), _p(beta),
                               *[_p(cache[n]) for n in ["S_b", "R", "kbuf", "vbuf", "abuf", "bbuf", "pos", "rscale"]],
                               N, H, dk, dv, C, _p(o))
    if rc:
        raise RuntimeError(f"sched_decode_step failed ({rc})")
    return o


def to_bf16_bits(x):
    """Round fp32 values to bf16 (nearest-even); returns uint16 bits."""
    lib = _load()
    x = _c(x, np.float32)
    y = np.zeros(x.shape, np.uint16)
    lib.sched_f32_to_bf16(_p(x), _p(y), x.size)
    return y


def schedule_tok_from_states(q, k, v, alpha, beta, states, cu_seqlens, C):
    """fp32 schedule model of P_tok, started from the given boundary states
    (chunk_states layout).  Returns (o [T,H,dv] fp32 before the output cast,
    R_final [N,H,dv,dk], Rs_final [N,H]): the running state Rs * R after each
    sequence's last token."""
    lib = _load()
    if not hasattr(lib, "_tok_states_ready"):
        P, i32 = ctypes.c_void_p, ctypes.c_int32
        lib.sched_tok_from_states.restype = ctypes.c_int
        lib.sched_tok_from_states.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, P, P, P]
        lib._tok_states_ready = True
    q, k, v = _c(q, np.float32), _c(k, np.float32), _c(v, np.float32)
    alpha, beta = _c(alpha, np.float32), _c(beta, np.float32)
    states = _c(states, np.float32)
    cu = _c(cu_seqlens, np.int32)
    T, H, dk = k.shape
    dv = v.shape[2]
    N = cu.shape[0] - 1
    o = np.zeros((T, H, dv), np.float32)
    Rf = np.zeros((N, H, dv, dk), np.float32)
    Rs = np.zeros((N, H), np.float32)
    rc = lib.sched_tok_from_states(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(states), _p(cu),
                                   N, H, dk, dv, C, _p(o), _p(Rf), _p(Rs))
    if rc:
        raise RuntimeError(f"sched_tok_from_states failed ({rc})")
    return o, Rf, Rs
