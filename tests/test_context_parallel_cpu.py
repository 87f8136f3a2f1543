"""Context-parallel hand-off of one long sequence over gloo ranks on CPU.

Each rank runs the fp32 schedule model (the bit-level model of the CUDA
schedule) on its chunk-aligned part, starting from the state the previous rank
sent.  Concatenated, the parts must equal the unsplit forward bit for bit:
splitting at a chunk boundary changes no result.

The backward hand-off runs in reverse rank order with the fp64 adjoint as the
per-rank backward (from the fp32 boundary state the forward handed over).
Concatenated, the parts match the unsplit fp64 adjoint to within the fp32
rounding of those boundary states.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from gated_deltanet_cpr_delta_b200 import context_parallel as cp
from gated_deltanet_cpr_delta_b200 import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _model_forward(q, k, v, alpha, beta, C, state_in):
    T = q.shape[0]
    si = None if state_in is None else state_in.numpy()
    m = oracle.schedule_forward(q.numpy(), k.numpy(), v.numpy(), alpha.numpy(), beta.numpy(),
                                np.array([0, T], np.int32), C, state_in=si)
    return torch.from_numpy(np.ascontiguousarray(m["o"])), torch.from_numpy(np.ascontiguousarray(m["states"]))


def _worker(rank, world, port, L, C, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = synth.make_batch(70, [L], 2, 16, 16, "bf16")
        S0 = synth.bf16_values(np.random.default_rng(71).standard_normal((1, 2, 16, 16)).astype(np.float32))
        s = cp.split_points(L, C, world)
        a0, a1 = s[rank], s[rank + 1]
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x[a0:a1]))
        o, st, s2 = cp.cp_forward(t(b.q), t(b.k), t(b.v), t(b.alpha), t(b.beta), C, L, forward=_model_forward,
                                  state_in=torch.from_numpy(S0) if rank == 0 else None)
        out[rank] = (o.numpy(), st.numpy(), s2)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,L,C", [(2, 5 * 16 + 7, 16), (3, 9 * 16, 16), (3, 40, 16)])
def test_context_parallel_hand_off_is_bitwise_unsplit(world, L, C):
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), L, C, out), nprocs=world, join=True)
    parts = [out[r] for r in range(world)]
    assert all(p[2] == parts[0][2] for p in parts)
    s = parts[0][2]
    assert s[0] == 0 and s[-1] == L and all(x % C == 0 for x in s[:-1]) and s == sorted(s)
    o, st = cp.gather_unsplit([torch.from_numpy(p[0]) for p in parts], [torch.from_numpy(p[1]) for p in parts])
    b = synth.make_batch(70, [L], 2, 16, 16, "bf16")
    S0 = synth.bf16_values(np.random.default_rng(71).standard_normal((1, 2, 16, 16)).astype(np.float32))
    full = oracle.schedule_forward(b.q, b.k, b.v, b.alpha, b.beta, b.cu_seqlens, C, state_in=S0)
    assert np.array_equal(o.numpy().view(np.uint32), full["o"].view(np.uint32))
    assert np.array_equal(st.numpy().view(np.uint32), full["states"].view(np.uint32))


def test_split_points():
    assert cp.split_points(5 * 16 + 7, 16, 2) == [0, 32, 87]
    assert cp.split_points(100, 64, 3) == [0, 0, 0, 100]
    assert cp.split_points(4096, 64, 8) == [0, 512, 1024, 1536, 2048, 2560, 3072, 3584, 4096]
    with pytest.raises(ValueError):
        cp.split_points(10, 0, 2)


def _oracle_backward(q, k, v, alpha, beta, dO, chunk_states, C, dstate_out):
    T = q.shape[0]
    g = oracle.adjoint(q.numpy(), k.numpy(), v.numpy(), alpha.numpy(), beta.numpy(), dO.numpy(),
                       np.array([0, T], np.int32), C, state_in=chunk_states[:1].numpy(),
                       dstate_out=None if dstate_out is None else dstate_out.numpy())
    return tuple(torch.from_numpy(np.ascontiguousarray(g[n]).astype(np.float32))
                 for n in ("dq", "dk", "dv", "dalpha", "dbeta", "dstate_in"))


def _bwd_worker(rank, world, port, L, C, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = synth.make_batch(72, [L], 2, 16, 16, "f32")
        rng = np.random.default_rng(73)
        S0 = (rng.standard_normal((1, 2, 16, 16)) * 0.3).astype(np.float32)
        W = (rng.standard_normal((1, 2, 16, 16)) * 0.1).astype(np.float32)
        dO = (rng.standard_normal((L, 2, 16)) * 0.5).astype(np.float32)
        s = cp.split_points(L, C, world)
        a0, a1 = s[rank], s[rank + 1]
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x[a0:a1]))
        _, st, _ = cp.cp_forward(t(b.q), t(b.k), t(b.v), t(b.alpha), t(b.beta), C, L, forward=_model_forward,
                                 state_in=torch.from_numpy(S0) if rank == 0 else None)
        g = cp.cp_backward(t(b.q), t(b.k), t(b.v), t(b.alpha), t(b.beta), t(dO), st, C, L,
                           backward=_oracle_backward,
                           dstate_out=torch.from_numpy(W) if rank == world - 1 else None)
        out[rank] = tuple(x.numpy() for x in g)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,L,C", [(2, 5 * 16 + 7, 16), (3, 9 * 16, 16), (3, 40, 16)])
def test_context_parallel_backward_hand_off(world, L, C):
    out = mp.Manager().dict()
    mp.spawn(_bwd_worker, args=(world, _free_port(), L, C, out), nprocs=world, join=True)
    parts = [out[r] for r in range(world)]
    b = synth.make_batch(72, [L], 2, 16, 16, "f32")
    rng = np.random.default_rng(73)
    S0 = (rng.standard_normal((1, 2, 16, 16)) * 0.3).astype(np.float32)
    W = (rng.standard_normal((1, 2, 16, 16)) * 0.1).astype(np.float32)
    dO = (rng.standard_normal((L, 2, 16)) * 0.5).astype(np.float32)
    ref = oracle.adjoint(b.q, b.k, b.v, b.alpha, b.beta, dO, np.array([0, L], np.int32), C, state_in=S0,
                         dstate_out=W)
    for i, name in enumerate(("dq", "dk", "dv", "dalpha", "dbeta")):
        got = np.concatenate([p[i] for p in parts])
        scale = max(np.max(np.abs(ref[name])), 1e-3)
        assert np.max(np.abs(got - ref[name])) <= 1e-5 * scale, name
    scale = max(np.max(np.abs(ref["dstate_in"])), 1e-3)
    assert np.max(np.abs(parts[0][5] - ref["dstate_in"])) <= 1e-5 * scale
