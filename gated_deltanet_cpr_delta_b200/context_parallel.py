"""Context parallelism for one long sequence: the boundary state is handed from
rank to rank at chunk-aligned split points, point to point.

Rank r owns tokens [s_r, s_{r+1}) of the sequence, every s_r a multiple of the
chunk size C.  Its forward starts from the state at s_r, which rank r-1
computes and sends (one d_v x d_k fp32 state per head).  Splitting a sequence
at a chunk boundary gives the same bits as not splitting it: the boundary
states of the parts are the boundary states of the whole, and every output
comes from the per-token recurrence started at its chunk's boundary state
(IsoExec summary page, "Chunkwise-Parallel Recurrent (CPR) Gated DeltaNet").
So the hand-off changes no result.  The boundary chain stays serial across
ranks: this spreads the sequence's memory and its parallel work over the GPUs,
not the serial scan.

The backward runs the same split in reverse rank order.  Rank r needs the
loss gradient for its last state (the state at s_{r+1}); rank r+1 computes it
as its dstate_in and sends it back.  The library's backward takes it as
dstate_out.  A split at a chunk boundary gives the same bits as the unsplit
backward here too.

`forward` / `backward` are the per-rank calls: by default the library's
gdn_cpr_forward / gdn_cpr_backward on the current CUDA device.  A caller may
pass other implementations with the same meaning; the CPU tests pass the fp32
schedule model and the fp64 adjoint.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def split_points(L: int, C: int, world: int) -> List[int]:
    """Chunk-aligned split of L tokens over `world` ranks: s_0 = 0 <= s_1 <= ...
    <= s_world = L, every interior s_r = C * floor(r * floor(L/C) / world).  The
    full chunks are shared out as evenly as they go; the partial last chunk, if
    any, goes to the last rank."""
    if L < 0 or C <= 0 or world <= 0:
        raise ValueError("bad split arguments")
    nfull = L // C
    return [0] + [C * (nfull * r // world) for r in range(1, world)] + [L]


def _library_forward(q, k, v, alpha, beta, C, state_in):
    from . import gdn
    T = q.shape[0]
    cu = torch.tensor([0, T], dtype=torch.int32, device=q.device)
    o, states = gdn.gdn_cpr_forward(q, k, v, alpha, beta, cu, C, cu_seqlens_host=[0, T], state_in=state_in)
    return o, states


def cp_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor, beta: torch.Tensor, C: int,
               L: int, group=None, forward: Optional[Callable] = None,
               state_in: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor, List[int]]:
    """This rank's part of a context-parallel CPR forward of one sequence of L
    tokens.  q, k, v, alpha, beta hold only this rank's tokens
    [s_r, s_{r+1}) with s = split_points(L, C, world) ([T_r, H, d] and [T_r, H]).
    state_in ([1, H, d_v, d_k] fp32, rank 0 only) is the state at token 0.

    Returns (o of this rank's tokens, this rank's chunk states, s).  The chunk
    states of rank r are the states at s_r, s_r + C, ..., s_r + floor(T_r/C)*C;
    dropping each later rank's first entry (the state it received) and
    concatenating gives the unsplit forward's chunk states."""
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    s = split_points(L, C, world)
    T_r = s[rank + 1] - s[rank]
    if q.shape[0] != T_r:
        raise ValueError(f"rank {rank} holds {q.shape[0]} tokens, its split is {T_r}")
    fwd = forward or _library_forward
    H, dv, dk = v.shape[1], v.shape[2], k.shape[2]
    if rank > 0:
        incoming = torch.empty(1, H, dv, dk, dtype=torch.float32, device=q.device)
        dist.recv(incoming, src=dist.get_global_rank(group, rank - 1) if group is not None else rank - 1, group=group)
        state_in = incoming
    o, states = fwd(q, k, v, alpha, beta, C, state_in)
    if rank + 1 < world:
        # this rank's last chunk state is the state at s_{r+1} (T_r is a multiple of C here)
        out = states[-1:].contiguous()
        dist.send(out, dst=dist.get_global_rank(group, rank + 1) if group is not None else rank + 1, group=group)
    return o, states, s


def _library_backward(q, k, v, alpha, beta, dO, chunk_states, C, dstate_out):
    from . import gdn
    T = q.shape[0]
    cu = torch.tensor([0, T], dtype=torch.int32, device=q.device)
    return gdn.gdn_cpr_backward(q, k, v, alpha, beta, dO, chunk_states, cu, C, cu_seqlens_host=[0, T],
                                dstate_out=dstate_out)


def cp_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor, beta: torch.Tensor,
                dO: torch.Tensor, chunk_states: torch.Tensor, C: int, L: int, group=None,
                backward: Optional[Callable] = None, dstate_out: Optional[torch.Tensor] = None):
    """This rank's part of the context-parallel backward of one sequence split
    as in :func:`cp_forward`.  q, k, v, alpha, beta, dO hold this rank's tokens;
    chunk_states are this rank's chunk states from cp_forward.  dstate_out
    ([1, H, d_v, d_k] fp32, last rank only, or None) is the loss gradient for
    the sequence's final state.

    The last rank runs first.  Each rank receives the gradient for its last
    state from rank r+1, runs its backward and sends its dstate_in to rank r-1.
    Returns this rank's (dq, dk, dv, dalpha, dbeta, dstate_in); rank 0's
    dstate_in is the gradient for the sequence's state_in."""
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    s = split_points(L, C, world)
    T_r = s[rank + 1] - s[rank]
    if q.shape[0] != T_r:
        raise ValueError(f"rank {rank} holds {q.shape[0]} tokens, its split is {T_r}")
    bwd = backward or _library_backward
    H, dv, dk = v.shape[1], v.shape[2], k.shape[2]
    if rank + 1 < world:
        incoming = torch.empty(1, H, dv, dk, dtype=torch.float32, device=q.device)
        dist.recv(incoming, src=dist.get_global_rank(group, rank + 1) if group is not None else rank + 1, group=group)
        dstate_out = incoming
    grads = bwd(q, k, v, alpha, beta, dO, chunk_states, C, dstate_out)
    if rank > 0:
        dist.send(grads[5].contiguous(), dst=dist.get_global_rank(group, rank - 1) if group is not None else rank - 1,
                  group=group)
    return grads


def gather_unsplit(parts_o: Sequence[torch.Tensor], parts_states: Sequence[torch.Tensor]):
    """Concatenate per-rank results into the unsplit forward's (o, chunk states)."""
    o = torch.cat(list(parts_o))
    st = torch.cat([parts_states[0]] + [p[1:] for p in parts_states[1:]])
    return o, st
