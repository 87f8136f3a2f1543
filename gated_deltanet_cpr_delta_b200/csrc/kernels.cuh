// kernels.cuh -- CUDA kernels of the CPR Gated DeltaNet path (sm_100a).
//
// Method: the gated delta rule evaluated chunkwise-parallel recurrent (CPR),
// IsoExec summary page, section "Chunkwise-Parallel Recurrent (CPR) Gated
// DeltaNet".  Outputs come from the per-token recurrence (P_tok) started at
// each chunk-boundary state.  Boundary states come from the chunk-level update
// P_chunk.  Decode runs P_tok and re-synchronises with P_chunk every C tokens.
//
// Kernels, in forward order:
//   k_tables    per-sequence offsets from the device cu_seqlens (+ validation)
//   k_prep      P_chunk part 1 per full chunk and head: decays D, Gram, w, u0
//   k_chain     P_chunk part 2: boundary states, serial over one sequence's chunks
//   k_tok       P_tok over every chunk in parallel -> o (and the running cache state)
//   k_cache_fill decode cache for a continuation
// Decode: k_dec_tok (P_tok + append), then k_dec_resync (P_chunk at a boundary).
// Backward: k_bwd_scan (boundary adjoints, serial per sequence, head and row tile), k_bgrad (per chunk, tcgen05).
#pragma once

#include "k_tables.cuh"
#include "k_ptok.cuh"
#include "k_prep.cuh"
#include "k_pchunk.cuh"
#include "k_decode.cuh"
#include "k_bwd.cuh"
#include "k_bgrad.cuh"
