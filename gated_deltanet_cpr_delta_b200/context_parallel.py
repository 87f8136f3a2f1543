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

`forward` is the per-rank forward: by default the library's gdn_cpr_forward on
the current CUDA device; a caller may pass another implementation with the same
meaning (the CPU tests pass the fp32 schedule model).
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


def gather_unsplit(parts_o: Sequence[torch.Tensor], parts_states: Sequence[torch.Tensor]):
    """Concatenate per-rank results into the unsplit forward's (o, chunk states)."""
    o = torch.cat(list(parts_o))
    st = torch.cat([parts_states[0]] + [p[1:] for p in parts_states[1:]])
    return o, st
