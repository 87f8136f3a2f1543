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
#pragma once

#include "schedule.cuh"

namespace gdn {

// ------------------------------------------------------------------ tables
// One CTA.  For every sequence n (L_n = cu[n+1]-cu[n]):
//   cto[n] = sum_{m<n} ceil(L_m/C)      (chunk tasks of k_tok)
//   fco[n] = sum_{m<n} floor(L_m/C)     (full chunks: k_prep / k_chain)
//   so[n]  = sum_{m<n} (floor(L_m/C)+1) (chunk-state slots)
// and the totals at index N.  err[0] = 1 if the device cu_seqlens is invalid
// or disagrees with the host-derived totals; every later kernel then exits.
__global__ void k_tables(const int32_t* __restrict__ cu, int N, int C, int64_t T_total,
                         int64_t want_tasks, int64_t want_full, int64_t want_states,
                         int32_t* cto, int32_t* fco, int32_t* so, int32_t* err)
{
    __shared__ long long wsum[3][32];
    __shared__ long long tot[3];
    __shared__ int bad_any;
    const int tid = threadIdx.x, nth = blockDim.x;
    if (tid == 0) bad_any = 0;
    __syncthreads();
    const int per = (N + nth - 1) / nth;
    const int n0 = min(N, tid * per), n1 = min(N, n0 + per);
    long long a = 0, b = 0, c = 0;
    int bad = 0;
    for (int n = n0; n < n1; ++n) {
        const int L = cu[n + 1] - cu[n];
        if (L < 0) bad = 1;
        const int Lc = L < 0 ? 0 : L;
        a += (Lc + C - 1) / C;
        b += Lc / C;
        c += Lc / C + 1;
    }
    // block-wide exclusive scan of (a, b, c)
    const int lane = tid & 31, wid = tid >> 5;
    long long va = a, vb = b, vc = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const long long xa = __shfl_up_sync(kFullMask, va, d);
        const long long xb = __shfl_up_sync(kFullMask, vb, d);
        const long long xc = __shfl_up_sync(kFullMask, vc, d);
        if (lane >= d) { va += xa; vb += xb; vc += xc; }
    }
    if (lane == 31) { wsum[0][wid] = va; wsum[1][wid] = vb; wsum[2][wid] = vc; }
    __syncthreads();
    if (tid == 0) {
        long long ra = 0, rb = 0, rc = 0;
        for (int w = 0; w < (nth + 31) / 32; ++w) {
            const long long ta = wsum[0][w], tb = wsum[1][w], tc = wsum[2][w];
            wsum[0][w] = ra; wsum[1][w] = rb; wsum[2][w] = rc;
            ra += ta; rb += tb; rc += tc;
        }
        tot[0] = ra; tot[1] = rb; tot[2] = rc;
    }
    __syncthreads();
    long long ea = wsum[0][wid] + va - a, eb = wsum[1][wid] + vb - b, ec = wsum[2][wid] + vc - c;
    for (int n = n0; n < n1; ++n) {
        cto[n] = (int32_t)ea; fco[n] = (int32_t)eb; so[n] = (int32_t)ec;
        const int L = max(0, cu[n + 1] - cu[n]);
        ea += (L + C - 1) / C; eb += L / C; ec += L / C + 1;
    }
    if (bad) atomicOr(&bad_any, 1);
    __syncthreads();
    if (tid == 0) {
        cto[N] = (int32_t)tot[0]; fco[N] = (int32_t)tot[1]; so[N] = (int32_t)tot[2];
        const bool ok = !bad_any && cu[0] == 0 && (int64_t)cu[N] == T_total &&
                        tot[0] == want_tasks && tot[1] == want_full && tot[2] == want_states;
        err[0] = ok ? 0 : 1;
    }
}

// ------------------------------------------------------------------ P_tok
// Per-thread share of one state row in the P_tok kernels: 4 consecutive lanes
// own a row, lane p holds elements [p*EPT, (p+1)*EPT) = leaves 2p and 2p+1.
template <int DK>
struct RowSplit {
    static constexpr int TPR = 4;
    static constexpr int EPT = DK / TPR;
    static constexpr int L = DK / kLeaves;
    // smem row padding: keeps the 4 lanes' 16-byte reads in distinct banks
    static constexpr int PAD = EPT >= 16 ? 4 : 0;
    static constexpr int KS = DK + TPR * PAD;  // padded row stride (floats)
    __device__ static constexpr int off(int p) { return p * (EPT + PAD); }
    __device__ static constexpr int smem_index(int j) { return j + (j / EPT) * PAD; }
};

template <int N>
__device__ __forceinline__ void lds_vec(float (&r)[N], const float* s)
{
    static_assert(N % 4 == 0, "vector load");
#pragma unroll
    for (int e = 0; e < N; e += 4) {
        const float4 x = *reinterpret_cast<const float4*>(s + e);
        r[e] = x.x; r[e + 1] = x.y; r[e + 2] = x.z; r[e + 3] = x.w;
    }
}

// One P_tok step for this thread's share of a row.  kt/qt point at this
// thread's slice of k_t/q_t (smem).  Returns o_t[row] (same bits in all 4 lanes).
template <int DK>
__device__ __forceinline__ float ptok_step(float (&R)[DK / 4], const float* kt, const float* qt,
                                           float v_i, float a, float b)
{
    using RS = RowSplit<DK>;
    constexpr int L = RS::L;
    float kr[RS::EPT];
    lds_vec(kr, kt);
    const float u = tree_4lanes(leaf_dot<L>(R, kr), leaf_dot<L>(R + L, kr + L));
    const float d = fmul(b, fsub(v_i, fmul(a, u)));
#pragma unroll
    for (int e = 0; e < RS::EPT; ++e) R[e] = ffma(d, kr[e], fmul(a, R[e]));
    float qr[RS::EPT];
    lds_vec(qr, qt);
    return tree_4lanes(leaf_dot<L>(R, qr), leaf_dot<L>(R + L, qr + L));
}

template <int DK, int DV, int C>
struct TokCfg {
    using RS = RowSplit<DK>;
    static constexpr int RT = DV < 64 ? DV : 64;  // rows per CTA
    static constexpr int NT = DV / RT;            // row tiles per head
    static constexpr int THREADS = RT * RS::TPR;
    static constexpr size_t SMEM = sizeof(float) * (2 * C * RS::KS + 2 * C * RT + 2 * C);
};

// Stage `len` tokens of a [T,H,D] input (rows tok0.., head h) into smem rows of
// stride `ld`, widened to fp32; element j goes to column idx(j).
template <int D, typename IdxFn>
__device__ __forceinline__ void stage_rows(float* dst, int ld, const void* src, int64_t tok0, int len, int H,
                                           int h, int bf16, IdxFn idx)
{
    for (int e = threadIdx.x; e < len * (D / 8); e += blockDim.x) {
        const int t = e / (D / 8), j8 = (e % (D / 8)) * 8;
        float x[8];
        load8(src, ((tok0 + t) * H + h) * (int64_t)D + j8, bf16, x);
        float* d = dst + t * ld + idx(j8);
        *reinterpret_cast<float4*>(d) = make_float4(x[0], x[1], x[2], x[3]);
        *reinterpret_cast<float4*>(d + 4) = make_float4(x[4], x[5], x[6], x[7]);
    }
}

struct IdxIdentity {
    __device__ int operator()(int j) const { return j; }
};
template <int DK>
struct IdxRowSplit {
    __device__ int operator()(int j) const { return RowSplit<DK>::smem_index(j); }
};

// Intra-chunk recurrence: one CTA per (chunk task, head, row tile).
template <int DK, int DV, int C>
__global__ void __launch_bounds__(TokCfg<DK, DV, C>::THREADS)
k_tok(const void* __restrict__ q, const void* __restrict__ k, const void* __restrict__ v,
      const float* __restrict__ alpha, const float* __restrict__ beta,
      const int32_t* __restrict__ cu, const int32_t* __restrict__ cto, const int32_t* __restrict__ so,
      const int32_t* __restrict__ err, int N, int H, int in_bf16, int out_bf16,
      const float* __restrict__ states, void* __restrict__ o, float* __restrict__ cacheR)
{
    using Cf = TokCfg<DK, DV, C>;
    using RS = typename Cf::RS;
    if (__ldg(err)) return;
    extern __shared__ float4 smem_f4[];
    float* ks = reinterpret_cast<float*>(smem_f4);
    float* qs = ks + C * RS::KS;
    float* vs = qs + C * RS::KS;
    float* os = vs + C * Cf::RT;
    float* as = os + C * Cf::RT;
    float* bs = as + C;

    const int r = blockIdx.x % Cf::NT;
    const int gh = blockIdx.x / Cf::NT;
    const int h = gh % H;
    const int g = gh / H;
    const int n = find_seq(cto, N, g);
    const int c = g - __ldg(cto + n);
    const int seq0 = __ldg(cu + n);
    const int Ln = __ldg(cu + n + 1) - seq0;
    const int64_t tok0 = (int64_t)seq0 + (int64_t)c * C;
    const int len = min(C, Ln - c * C);
    const int64_t slot = (int64_t)__ldg(so + n) + c;

    stage_rows<DK>(ks, RS::KS, k, tok0, len, H, h, in_bf16, IdxRowSplit<DK>());
    stage_rows<DK>(qs, RS::KS, q, tok0, len, H, h, in_bf16, IdxRowSplit<DK>());
    for (int e = threadIdx.x; e < len * (Cf::RT / 8); e += blockDim.x) {
        const int t = e / (Cf::RT / 8), i8 = (e % (Cf::RT / 8)) * 8;
        float x[8];
        load8(v, ((tok0 + t) * H + h) * (int64_t)DV + r * Cf::RT + i8, in_bf16, x);
#pragma unroll
        for (int m = 0; m < 8; ++m) vs[t * Cf::RT + i8 + m] = x[m];
    }
    for (int t = threadIdx.x; t < len; t += blockDim.x) {
        as[t] = __ldg(alpha + (tok0 + t) * H + h);
        bs[t] = __ldg(beta + (tok0 + t) * H + h);
    }

    const int row = threadIdx.x / RS::TPR, p = threadIdx.x % RS::TPR;
    const int64_t grow = (int64_t)r * Cf::RT + row;
    float R[RS::EPT];
    {
        const float* src = states + ((slot * H + h) * DV + grow) * DK + p * RS::EPT;
#pragma unroll
        for (int e = 0; e < RS::EPT; e += 4) {
            const float4 x = __ldg(reinterpret_cast<const float4*>(src + e));
            R[e] = x.x; R[e + 1] = x.y; R[e + 2] = x.z; R[e + 3] = x.w;
        }
    }
    __syncthreads();

    for (int t = 0; t < len; ++t) {
        const float ot = ptok_step<DK>(R, ks + t * RS::KS + RS::off(p), qs + t * RS::KS + RS::off(p),
                                       vs[t * Cf::RT + row], as[t], bs[t]);
        if (p == 0) os[t * Cf::RT + row] = ot;
    }

    if (cacheR != nullptr && len < C) {  // last, partial chunk: running state for decode
        float* dst = cacheR + (((int64_t)n * H + h) * DV + grow) * DK + p * RS::EPT;
#pragma unroll
        for (int e = 0; e < RS::EPT; e += 4)
            *reinterpret_cast<float4*>(dst + e) = make_float4(R[e], R[e + 1], R[e + 2], R[e + 3]);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < len * (Cf::RT / 8); e += blockDim.x) {
        const int t = e / (Cf::RT / 8), i8 = (e % (Cf::RT / 8)) * 8;
        store8(o, ((tok0 + t) * H + h) * (int64_t)DV + r * Cf::RT + i8, out_bf16, os + t * Cf::RT + i8);
    }
}

// ------------------------------------------------------------------ P_chunk
template <int DK, int DV, int C>
struct ChunkCfg {
    static constexpr int KS = DK + 4;      // padded k / w row stride
    static constexpr int C1 = C + 1;       // decay matrix row stride
    static constexpr int CT = C + 4;       // c^T row stride
    static constexpr int DCS = C + 4;      // stride of D[C][.] rows in the workspace
    static constexpr int RTB = DV < 32 ? DV : 32;  // boundary-state rows per tile
    static constexpr int NTB = DV / RTB;
    static constexpr int THREADS = 256;
};

// P_chunk part 1 for one chunk, by one CTA.  ks [C][KS], vs [C][DV], as/bs [C]
// in smem.  Dm [(C+1)^2] and cT [C][CT] are smem scratch.  Writes
//   w_t  -> wout[(t-1)*ldw + j],   u0_t -> uout[(t-1)*ldu + i],   D[C][s] -> dCout[s]
// (any address space).  uout may alias vs: each column of vs is read by the
// same thread that later writes that column of uout, and only before it does.
template <int DK, int DV, int C>
__device__ __forceinline__ void chunk_prep(const float* ks, const float* vs, const float* as, const float* bs,
                                           float* Dm, float* cT, float* wout, int ldw, float* uout, int ldu,
                                           float* dCout)
{
    using Cf = ChunkCfg<DK, DV, C>;
    constexpr int KS = Cf::KS, C1 = Cf::C1, CT = Cf::CT;
    // decay products D[t][s] = D[t-1][s] * alpha_t, D[s][s] = 1  (tokens 1..C)
    for (int s = threadIdx.x; s <= C; s += blockDim.x) {
        float d = 1.0f;
        Dm[s * C1 + s] = d;
        for (int t = s + 1; t <= C; ++t) {
            d = fmul(d, as[t - 1]);
            Dm[t * C1 + s] = d;
        }
    }
    __syncthreads();
    // c[t][s] = D[t][s] * tree(k_s, k_t), stored transposed: cT[s-1][t-1]
    for (int e = threadIdx.x; e < C * C; e += blockDim.x) {
        const int tau = e / C, sig = e % C;  // 0-based tokens, need sig < tau
        if (sig < tau) {
            const float G = tree_dot<DK>(ks + sig * KS, ks + tau * KS);
            cT[sig * CT + tau] = fmul(Dm[(tau + 1) * C1 + (sig + 1)], G);
        }
    }
    if (dCout != nullptr)
        for (int s = threadIdx.x; s <= C; s += blockDim.x) dCout[s] = Dm[C * C1 + s];
    __syncthreads();
    // forward substitution, one column per thread, right-looking: after token
    // s is final, its term enters every later token's chain.  For each token t
    // the chain still runs over s = 1..t-1 in ascending order.
    for (int col = threadIdx.x; col < DV + DK; col += blockDim.x) {
        float acc[C];
        const bool is_u = col < DV;
        const int j = is_u ? 0 : col - DV;
        if (is_u) {
#pragma unroll
            for (int tau = 0; tau < C; ++tau) acc[tau] = vs[tau * DV + col];
        } else {
#pragma unroll
            for (int tau = 0; tau < C; ++tau) acc[tau] = fmul(Dm[(tau + 1) * C1], ks[tau * KS + j]);
        }
#pragma unroll
        for (int sig = 0; sig < C; ++sig) {
            const float x = fmul(bs[sig], acc[sig]);
            if (is_u) uout[sig * ldu + col] = x;
            else wout[sig * ldw + j] = x;
#pragma unroll
            for (int tau = sig + 1; tau < C; ++tau) acc[tau] = ffma(-cT[sig * CT + tau], x, acc[tau]);
        }
    }
    __syncthreads();
}

// P_chunk part 2 on a tile of RTB boundary-state rows, by one CTA:
//   e_t[i] = D[C][t] * (u0_t[i] - tree(S_i, w_t)),
//   S_i,j <- chain_t fma(e_t[i], k_t[j], .) from D[C][0] * S_ij.
// Ss [RTB][KS], ws [C][KS], ks [C][KS], us [C][ldu], dCs [C+1], es [C][RTB] (scratch).
template <int DK, int RTB, int C>
__device__ __forceinline__ void chunk_advance(float* Ss, const float* ws, const float* us, int ldu,
                                              const float* ks, const float* dCs, float* es)
{
    constexpr int KS = DK + 4;
    for (int e = threadIdx.x; e < C * RTB; e += blockDim.x) {
        const int i = e % RTB, tau = e / RTB;
        const float sw = tree_dot<DK>(Ss + i * KS, ws + tau * KS);
        es[tau * RTB + i] = fmul(dCs[tau + 1], fsub(us[tau * ldu + i], sw));
    }
    __syncthreads();
    const float d0 = dCs[0];
    for (int e = threadIdx.x; e < RTB * DK; e += blockDim.x) {
        const int i = e / DK, j = e % DK;
        float acc = fmul(d0, Ss[i * KS + j]);
#pragma unroll 8
        for (int tau = 0; tau < C; ++tau) acc = ffma(es[tau * RTB + i], ks[tau * KS + j], acc);
        Ss[i * KS + j] = acc;  // only this thread reads or writes element (i, j) in this phase
    }
    __syncthreads();
}

template <int DK, int DV, int C>
struct PrepSmem {
    using Cf = ChunkCfg<DK, DV, C>;
    static constexpr int KS_OFF = 0;
    static constexpr int VS_OFF = KS_OFF + C * Cf::KS;
    static constexpr int DM_OFF = VS_OFF + C * DV;
    static constexpr int CT_OFF = DM_OFF + ((Cf::C1 * Cf::C1 + 3) / 4) * 4;
    static constexpr int AB_OFF = CT_OFF + C * Cf::CT;
    static constexpr size_t BYTES = sizeof(float) * (AB_OFF + 2 * C);
};

// P_chunk part 1 for every full chunk: one CTA per (full chunk, head).
template <int DK, int DV, int C>
__global__ void __launch_bounds__(256)
k_prep(const void* __restrict__ k, const void* __restrict__ v, const float* __restrict__ alpha,
       const float* __restrict__ beta, const int32_t* __restrict__ cu, const int32_t* __restrict__ fco,
       const int32_t* __restrict__ err, int N, int H, int in_bf16,
       float* __restrict__ w_ws, float* __restrict__ u_ws, float* __restrict__ dC_ws)
{
    using Cf = ChunkCfg<DK, DV, C>;
    using Sm = PrepSmem<DK, DV, C>;
    if (__ldg(err)) return;
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    float* ks = sm + Sm::KS_OFF;
    float* vs = sm + Sm::VS_OFF;
    float* Dm = sm + Sm::DM_OFF;
    float* cT = sm + Sm::CT_OFF;
    float* as = sm + Sm::AB_OFF;
    float* bs = as + C;

    const int task = blockIdx.x;
    const int h = task % H, g = task / H;
    const int n = find_seq(fco, N, g);
    const int64_t tok0 = (int64_t)__ldg(cu + n) + (int64_t)(g - __ldg(fco + n)) * C;
    stage_rows<DK>(ks, Cf::KS, k, tok0, C, H, h, in_bf16, IdxIdentity());
    stage_rows<DV>(vs, DV, v, tok0, C, H, h, in_bf16, IdxIdentity());
    for (int t = threadIdx.x; t < C; t += blockDim.x) {
        as[t] = __ldg(alpha + (tok0 + t) * H + h);
        bs[t] = __ldg(beta + (tok0 + t) * H + h);
    }
    __syncthreads();
    chunk_prep<DK, DV, C>(ks, vs, as, bs, Dm, cT, w_ws + (int64_t)task * C * DK, DK,
                          u_ws + (int64_t)task * C * DV, DV, dC_ws + (int64_t)task * Cf::DCS);
}

template <int DK, int DV, int C>
struct ChainSmem {
    using Cf = ChunkCfg<DK, DV, C>;
    static constexpr int SS_OFF = 0;
    static constexpr int WS_OFF = SS_OFF + Cf::RTB * Cf::KS;
    static constexpr int KS_OFF = WS_OFF + C * Cf::KS;
    static constexpr int US_OFF = KS_OFF + C * Cf::KS;
    static constexpr int ES_OFF = US_OFF + C * Cf::RTB;
    static constexpr int DC_OFF = ES_OFF + C * Cf::RTB;
    static constexpr size_t BYTES = sizeof(float) * (DC_OFF + Cf::DCS);
};

// Boundary states: one CTA per (sequence, head, row tile), serial over the
// sequence's full chunks.  Writes chunk_states[so[n] + c] for c = 0..floor(L/C).
template <int DK, int DV, int C>
__global__ void __launch_bounds__(256)
k_chain(const void* __restrict__ k, const float* __restrict__ state_in, const int32_t* __restrict__ cu,
        const int32_t* __restrict__ fco, const int32_t* __restrict__ so, const int32_t* __restrict__ err,
        int N, int H, int in_bf16, const float* __restrict__ w_ws, const float* __restrict__ u_ws,
        const float* __restrict__ dC_ws, float* __restrict__ states)
{
    using Cf = ChunkCfg<DK, DV, C>;
    using Sm = ChainSmem<DK, DV, C>;
    constexpr int KS = Cf::KS, RTB = Cf::RTB;
    if (__ldg(err)) return;
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    float* Ss = sm + Sm::SS_OFF;
    float* ws = sm + Sm::WS_OFF;
    float* ks = sm + Sm::KS_OFF;
    float* us = sm + Sm::US_OFF;
    float* es = sm + Sm::ES_OFF;
    float* dCs = sm + Sm::DC_OFF;

    const int r = blockIdx.x % Cf::NTB;
    const int nh = blockIdx.x / Cf::NTB;
    const int h = nh % H, n = nh / H;
    const int seq0 = __ldg(cu + n);
    const int nfull = (__ldg(cu + n + 1) - seq0) / C;
    const int64_t slot0 = __ldg(so + n);
    const int64_t g0 = __ldg(fco + n);
    const int64_t row0 = (int64_t)r * RTB;

    for (int e = threadIdx.x; e < RTB * (DK / 4); e += blockDim.x) {
        const int i = e / (DK / 4), j4 = (e % (DK / 4)) * 4;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (state_in != nullptr)
            x = __ldg(reinterpret_cast<const float4*>(state_in + (((int64_t)n * H + h) * DV + row0 + i) * DK + j4));
        *reinterpret_cast<float4*>(Ss + i * KS + j4) = x;
        *reinterpret_cast<float4*>(states + ((slot0 * H + h) * DV + row0 + i) * DK + j4) = x;
    }
    for (int c = 0; c < nfull; ++c) {
        __syncthreads();
        const int64_t task = (g0 + c) * H + h;
        const float* wsrc = w_ws + task * C * DK;
        for (int e = threadIdx.x; e < C * (DK / 4); e += blockDim.x) {
            const int t = e / (DK / 4), j4 = (e % (DK / 4)) * 4;
            *reinterpret_cast<float4*>(ws + t * KS + j4) = __ldg(reinterpret_cast<const float4*>(wsrc + t * DK + j4));
        }
        stage_rows<DK>(ks, KS, k, (int64_t)seq0 + (int64_t)c * C, C, H, h, in_bf16, IdxIdentity());
        const float* usrc = u_ws + task * C * DV + row0;
        for (int e = threadIdx.x; e < C * RTB; e += blockDim.x) {
            const int t = e / RTB, i = e % RTB;
            us[t * RTB + i] = __ldg(usrc + t * DV + i);
        }
        for (int s = threadIdx.x; s <= C; s += blockDim.x) dCs[s] = __ldg(dC_ws + task * Cf::DCS + s);
        __syncthreads();
        chunk_advance<DK, RTB, C>(Ss, ws, us, RTB, ks, dCs, es);
        float* dst = states + (((slot0 + c + 1) * H + h) * DV + row0) * DK;
        for (int e = threadIdx.x; e < RTB * (DK / 4); e += blockDim.x) {
            const int i = e / (DK / 4), j4 = (e % (DK / 4)) * 4;
            *reinterpret_cast<float4*>(dst + (int64_t)i * DK + j4) = *reinterpret_cast<const float4*>(Ss + i * KS + j4);
        }
    }
}

// Decode cache for a continuation: one CTA per (sequence, head).
template <int DK, int DV, int C>
__global__ void __launch_bounds__(256)
k_cache_fill(const void* __restrict__ k, const void* __restrict__ v, const float* __restrict__ alpha,
             const float* __restrict__ beta, const int32_t* __restrict__ cu, const int32_t* __restrict__ so,
             const int32_t* __restrict__ err, int N, int H, int in_bf16, const float* __restrict__ states,
             float* S_b, float* R, void* kbuf, void* vbuf, float* abuf, float* bbuf, int32_t* pos)
{
    if (__ldg(err)) return;
    const int nh = blockIdx.x;
    const int n = nh / H, h = nh % H;
    const int seq0 = __ldg(cu + n);
    const int Ln = __ldg(cu + n + 1) - seq0;
    const int p = Ln % C;
    const int64_t last = (int64_t)__ldg(so + n) + Ln / C;
    const float4* src = reinterpret_cast<const float4*>(states + (last * H + h) * (int64_t)DV * DK);
    float4* sb = reinterpret_cast<float4*>(S_b + (int64_t)nh * DV * DK);
    float4* rr = reinterpret_cast<float4*>(R + (int64_t)nh * DV * DK);
    for (int e = threadIdx.x; e < DV * DK / 4; e += blockDim.x) {
        const float4 x = src[e];
        sb[e] = x;
        if (p == 0) rr[e] = x;  // at a boundary the running state is the boundary state
    }
    const int esz = in_bf16 ? 2 : 4;
    // the p tokens of the open chunk, raw copies in the input dtype
    for (int e = threadIdx.x; e < p * (DK * esz / 16); e += blockDim.x) {
        const int s = e / (DK * esz / 16), b16 = e % (DK * esz / 16);
        const int64_t tok = (int64_t)seq0 + Ln - p + s;
        reinterpret_cast<uint4*>(kbuf)[((int64_t)nh * C + s) * (DK * esz / 16) + b16] =
            __ldg(reinterpret_cast<const uint4*>(k) + (tok * H + h) * (DK * esz / 16) + b16);
    }
    for (int e = threadIdx.x; e < p * (DV * esz / 16); e += blockDim.x) {
        const int s = e / (DV * esz / 16), b16 = e % (DV * esz / 16);
        const int64_t tok = (int64_t)seq0 + Ln - p + s;
        reinterpret_cast<uint4*>(vbuf)[((int64_t)nh * C + s) * (DV * esz / 16) + b16] =
            __ldg(reinterpret_cast<const uint4*>(v) + (tok * H + h) * (DV * esz / 16) + b16);
    }
    for (int s = threadIdx.x; s < p; s += blockDim.x) {
        const int64_t tok = (int64_t)seq0 + Ln - p + s;
        abuf[(int64_t)nh * C + s] = __ldg(alpha + tok * H + h);
        bbuf[(int64_t)nh * C + s] = __ldg(beta + tok * H + h);
    }
    if (threadIdx.x == 0) pos[nh] = p;
}

// ------------------------------------------------------------------ decode
template <int DK, int DV>
struct DecCfg {
    using RS = RowSplit<DK>;
    static constexpr int THREADS = DV * RS::TPR;
};

// One decode token per (sequence, head): P_tok on the running state R, append
// the token to the buffer, pos += 1 (pos == C marks a pending resync).
template <int DK, int DV, int C>
__global__ void __launch_bounds__(DecCfg<DK, DV>::THREADS)
k_dec_tok(const void* __restrict__ q, const void* __restrict__ k, const void* __restrict__ v,
          const float* __restrict__ alpha, const float* __restrict__ beta, int H, int in_bf16, int out_bf16,
          float* R, void* kbuf, void* vbuf, float* abuf, float* bbuf, int32_t* pos, void* __restrict__ o)
{
    using RS = RowSplit<DK>;
    __shared__ __align__(16) float ks[RS::KS];
    __shared__ __align__(16) float qs[RS::KS];
    __shared__ __align__(16) float vs[DV];
    const int nh = blockIdx.x;
    const int p = pos[nh];
    if (p < 0 || p >= C) return;
    stage_rows<DK>(ks, RS::KS, k, nh, 1, 1, 0, in_bf16, IdxRowSplit<DK>());
    stage_rows<DK>(qs, RS::KS, q, nh, 1, 1, 0, in_bf16, IdxRowSplit<DK>());
    stage_rows<DV>(vs, DV, v, nh, 1, 1, 0, in_bf16, IdxIdentity());
    const float a = __ldg(alpha + nh), b = __ldg(beta + nh);
    const int row = threadIdx.x / RS::TPR, part = threadIdx.x % RS::TPR;
    float* Rrow = R + ((int64_t)nh * DV + row) * DK + part * RS::EPT;
    float Rr[RS::EPT];
#pragma unroll
    for (int e = 0; e < RS::EPT; e += 4) {
        const float4 x = *reinterpret_cast<const float4*>(Rrow + e);
        Rr[e] = x.x; Rr[e + 1] = x.y; Rr[e + 2] = x.z; Rr[e + 3] = x.w;
    }
    __syncthreads();
    const float ot = ptok_step<DK>(Rr, ks + RS::off(part), qs + RS::off(part), vs[row], a, b);
#pragma unroll
    for (int e = 0; e < RS::EPT; e += 4)
        *reinterpret_cast<float4*>(Rrow + e) = make_float4(Rr[e], Rr[e + 1], Rr[e + 2], Rr[e + 3]);
    if (part == 0) store1(o, (int64_t)nh * DV + row, out_bf16, ot);
    // append the raw token to the buffer at slot p
    const int esz = in_bf16 ? 2 : 4;
    for (int e = threadIdx.x; e < DK * esz / 16; e += blockDim.x)
        reinterpret_cast<uint4*>(kbuf)[((int64_t)nh * C + p) * (DK * esz / 16) + e] =
            __ldg(reinterpret_cast<const uint4*>(k) + (int64_t)nh * (DK * esz / 16) + e);
    for (int e = threadIdx.x; e < DV * esz / 16; e += blockDim.x)
        reinterpret_cast<uint4*>(vbuf)[((int64_t)nh * C + p) * (DV * esz / 16) + e] =
            __ldg(reinterpret_cast<const uint4*>(v) + (int64_t)nh * (DV * esz / 16) + e);
    if (threadIdx.x == 0) {
        abuf[(int64_t)nh * C + p] = a;
        bbuf[(int64_t)nh * C + p] = b;
    }
    __syncthreads();  // every thread has read pos before it moves
    if (threadIdx.x == 0) pos[nh] = p + 1;
}

template <int DK, int DV, int C>
struct ResyncSmem {
    using Cf = ChunkCfg<DK, DV, C>;
    static constexpr int KS_OFF = 0;
    static constexpr int VS_OFF = KS_OFF + C * Cf::KS;
    static constexpr int WS_OFF = VS_OFF + C * DV;
    static constexpr int DM_OFF = WS_OFF + C * Cf::KS;
    static constexpr int CT_OFF = DM_OFF + ((Cf::C1 * Cf::C1 + 3) / 4) * 4;
    static constexpr int SS_OFF = CT_OFF + C * Cf::CT;
    static constexpr int ES_OFF = SS_OFF + Cf::RTB * Cf::KS;
    static constexpr int AB_OFF = ES_OFF + C * Cf::RTB;
    static constexpr int DC_OFF = AB_OFF + 2 * C;
    static constexpr size_t BYTES = sizeof(float) * (DC_OFF + Cf::DCS);
};

// Resync: for every (sequence, head) whose buffer holds C tokens (pos == C),
// S_b <- P_chunk(S_b, buffer), R <- S_b, pos <- 0.  Other CTAs exit at once.
template <int DK, int DV, int C>
__global__ void __launch_bounds__(256)
k_dec_resync(int in_bf16, float* S_b, float* R, const void* kbuf, const void* vbuf, const float* abuf,
             const float* bbuf, int32_t* pos)
{
    using Cf = ChunkCfg<DK, DV, C>;
    using Sm = ResyncSmem<DK, DV, C>;
    constexpr int KS = Cf::KS, RTB = Cf::RTB;
    const int nh = blockIdx.x;
    if (pos[nh] != C) return;
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    float* ks = sm + Sm::KS_OFF;
    float* vs = sm + Sm::VS_OFF;
    float* ws = sm + Sm::WS_OFF;
    float* Dm = sm + Sm::DM_OFF;
    float* cT = sm + Sm::CT_OFF;
    float* Ss = sm + Sm::SS_OFF;
    float* es = sm + Sm::ES_OFF;
    float* as = sm + Sm::AB_OFF;
    float* bs = as + C;
    float* dCs = sm + Sm::DC_OFF;

    // buffer rows are [nh][slot][D]: a [T, H=1, D] tensor starting at token nh*C
    stage_rows<DK>(ks, KS, kbuf, (int64_t)nh * C, C, 1, 0, in_bf16, IdxIdentity());
    stage_rows<DV>(vs, DV, vbuf, (int64_t)nh * C, C, 1, 0, in_bf16, IdxIdentity());
    for (int t = threadIdx.x; t < C; t += blockDim.x) {
        as[t] = abuf[(int64_t)nh * C + t];
        bs[t] = bbuf[(int64_t)nh * C + t];
    }
    __syncthreads();
    chunk_prep<DK, DV, C>(ks, vs, as, bs, Dm, cT, ws, KS, vs, DV, dCs);  // u0 overwrites v in place
    for (int r = 0; r < Cf::NTB; ++r) {
        float* Sg = S_b + ((int64_t)nh * DV + r * RTB) * DK;
        float* Rg = R + ((int64_t)nh * DV + r * RTB) * DK;
        for (int e = threadIdx.x; e < RTB * (DK / 4); e += blockDim.x) {
            const int i = e / (DK / 4), j4 = (e % (DK / 4)) * 4;
            *reinterpret_cast<float4*>(Ss + i * KS + j4) = *reinterpret_cast<const float4*>(Sg + (int64_t)i * DK + j4);
        }
        __syncthreads();
        chunk_advance<DK, RTB, C>(Ss, ws, vs + r * RTB, DV, ks, dCs, es);
        for (int e = threadIdx.x; e < RTB * (DK / 4); e += blockDim.x) {
            const int i = e / (DK / 4), j4 = (e % (DK / 4)) * 4;
            const float4 x = *reinterpret_cast<const float4*>(Ss + i * KS + j4);
            *reinterpret_cast<float4*>(Sg + (int64_t)i * DK + j4) = x;
            *reinterpret_cast<float4*>(Rg + (int64_t)i * DK + j4) = x;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) pos[nh] = 0;
}

}  // namespace gdn
