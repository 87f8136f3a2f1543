"""Seeded synthetic inputs for the CPR Gated DeltaNet layer.

This module only draws and shapes inputs; it contains none of the layer's
arithmetic.  Tests, the benchmark and the smoke check all take their inputs
from here, so the CUDA path and the CPU oracle see identical values.

Recipe (every sequence has its own stream, so a sequence's content does not
depend on its batch position or on the other sequences):

* varlen only: lengths = ``default_rng(seed).integers(lo, hi + 1, N)``;
* sequence ``n`` draws, from ``default_rng([seed, n])``, in this order,
  standard normals in fp64: ``x_q [L,H,dk]``, ``x_k [L,H,dk]``,
  ``x_v [L,H,dv]``, ``x_a [L,H]``, ``x_b [L,H]``;
* q, k: per-token, per-head L2 normalisation in fp64; v as drawn;
  q, k, v -> fp32 (round to nearest even) -> bf16 (nearest even) when the
  input dtype is bf16;
* alpha = exp(-softplus(x_a)), beta = sigmoid(x_b), in fp64, -> fp32.

These stand in for the activations of a hybrid-attention LLM's GDN layers
(no dataset or weights are involved).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    one, sh = np.uint32(1), np.uint32(16)
    u = (u + np.uint32(0x7FFF) + ((u >> sh) & one)) >> sh
    return u.astype(np.uint16)


def bf16_values(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 and return them widened back to fp32."""
    return (bf16_bits(x).astype(np.uint32) << 16).view(np.float32)


def _l2n(x: np.ndarray) -> np.ndarray:
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True))


def sequence_inputs(seed: int, n: int, L: int, H: int, dk: int, dv: int, dtype: str) -> Dict[str, np.ndarray]:
    """Inputs of sequence ``n`` (length L) of the seeded workload ``seed``."""
    rng = np.random.default_rng([seed, n])
    xq = rng.standard_normal((L, H, dk))
    xk = rng.standard_normal((L, H, dk))
    xv = rng.standard_normal((L, H, dv))
    xa = rng.standard_normal((L, H))
    xb = rng.standard_normal((L, H))
    q = _l2n(xq).astype(np.float32)
    k = _l2n(xk).astype(np.float32)
    v = xv.astype(np.float32)
    if dtype == "bf16":
        q, k, v = bf16_values(q), bf16_values(k), bf16_values(v)
    elif dtype != "f32":
        raise ValueError(dtype)
    alpha = np.exp(-np.logaddexp(0.0, xa)).astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-xb))).astype(np.float32)
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta)


@dataclass
class Batch:
    """A packed varlen batch. q,k [T,H,dk], v [T,H,dv] hold fp32 values (exact
    bf16 values when dtype == 'bf16'); alpha, beta [T,H] fp32."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    alpha: np.ndarray
    beta: np.ndarray
    cu_seqlens: np.ndarray
    dtype: str
    seq_ids: List[int] = field(default_factory=list)

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.cu_seqlens)

    @property
    def H(self) -> int:
        return self.k.shape[1]

    @property
    def dk(self) -> int:
        return self.k.shape[2]

    @property
    def dv(self) -> int:
        return self.v.shape[2]

    def subset(self, seqs: Sequence[int], heads: Optional[Sequence[int]] = None) -> "Batch":
        """The listed sequences (batch positions) and heads, re-packed."""
        heads = list(range(self.H)) if heads is None else list(heads)
        parts = {n: [] for n in ("q", "k", "v", "alpha", "beta")}
        lens = []
        for s in seqs:
            a, b = int(self.cu_seqlens[s]), int(self.cu_seqlens[s + 1])
            for n in parts:
                parts[n].append(getattr(self, n)[a:b][:, heads])
            lens.append(b - a)
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        return Batch(*(np.ascontiguousarray(np.concatenate(parts[n])) for n in parts), cu, self.dtype,
                     [self.seq_ids[s] for s in seqs] if self.seq_ids else list(seqs))


def make_batch(seed: int, lengths: Sequence[int], H: int, dk: int, dv: int, dtype: str,
               seq_ids: Optional[Sequence[int]] = None) -> Batch:
    """Pack sequences ``seq_ids`` (default 0..N-1) with the given lengths."""
    seq_ids = list(range(len(lengths))) if seq_ids is None else list(seq_ids)
    seqs = [sequence_inputs(seed, n, int(L), H, dk, dv, dtype) for n, L in zip(seq_ids, lengths)]
    cat = {n: np.ascontiguousarray(np.concatenate([s[n] for s in seqs])) for n in seqs[0]}
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return Batch(cat["q"], cat["k"], cat["v"], cat["alpha"], cat["beta"], cu, dtype, seq_ids)


def varlen_lengths(seed: int, N: int = 32, lo: int = 128, hi: int = 8192) -> List[int]:
    return [int(x) for x in np.random.default_rng(seed).integers(lo, hi + 1, N)]


# The workloads: name -> (seed, description).  Sizes are spelled out by the
# helpers below so that tests and the benchmark use the same numbers.
TINY = dict(seed=0, B=1, H=2, T=64, dk=16, dv=16, C=16, dtype="f32")
PREFILL = dict(seed=1, B=4, H=16, T=4096, dk=128, dv=128, C=64, dtype="bf16")
DECODE = dict(seed=2, B=64, H=32, T_prefill=2048, steps=256, dk=128, dv=128, C=64, dtype="bf16")
VARLEN = dict(seed=3, N=32, H=32, lo=128, hi=8192, dk=128, dv=128, C=64, dtype="bf16")
TRAIN = dict(seed=4, B=2, H=32, T=8192, dk=128, dv=128, C=64, dtype="bf16")


# ---------------------------------------------------------------- device recipe
# For the full-size workloads (up to ~150k tokens x 32 heads) the same recipe
# runs with torch on the GPU: sequence n uses a torch Philox generator seeded
# with seed * 1_000_003 + n, draws fp64 standard normals in the same order,
# and applies the same transforms.  The values differ from the numpy recipe
# (different bit generator) but have the same distribution.  Parity checks at
# these sizes copy the sampled sequences' inputs to the host for the oracle.
def make_batch_device(seed: int, lengths: Sequence[int], H: int, dk: int, dv: int, dtype: str,
                      device="cuda", seq_ids: Optional[Sequence[int]] = None):
    import torch

    seq_ids = list(range(len(lengths))) if seq_ids is None else list(seq_ids)
    tdt = {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]
    T = int(sum(lengths))
    q = torch.empty(T, H, dk, dtype=tdt, device=device)
    k = torch.empty(T, H, dk, dtype=tdt, device=device)
    v = torch.empty(T, H, dv, dtype=tdt, device=device)
    alpha = torch.empty(T, H, dtype=torch.float32, device=device)
    beta = torch.empty(T, H, dtype=torch.float32, device=device)
    a0 = 0
    for n, L in zip(seq_ids, lengths):
        L = int(L)
        g = torch.Generator(device=device)
        g.manual_seed(int(seed) * 1_000_003 + int(n))
        sl = slice(a0, a0 + L)
        xq = torch.randn(L, H, dk, dtype=torch.float64, device=device, generator=g)
        q[sl] = (xq / xq.norm(dim=-1, keepdim=True)).float().to(tdt)
        del xq
        xk = torch.randn(L, H, dk, dtype=torch.float64, device=device, generator=g)
        k[sl] = (xk / xk.norm(dim=-1, keepdim=True)).float().to(tdt)
        del xk
        v[sl] = torch.randn(L, H, dv, dtype=torch.float64, device=device, generator=g).float().to(tdt)
        xa = torch.randn(L, H, dtype=torch.float64, device=device, generator=g)
        xb = torch.randn(L, H, dtype=torch.float64, device=device, generator=g)
        alpha[sl] = torch.exp(-torch.logaddexp(torch.zeros_like(xa), xa)).float()
        beta[sl] = torch.sigmoid(xb).float()
        a0 += L
    cu_host = [0]
    for L in lengths:
        cu_host.append(cu_host[-1] + int(L))
    cu = torch.tensor(cu_host, dtype=torch.int32, device=device)
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta, cu_seqlens=cu, cu_host=cu_host, dtype=dtype)
