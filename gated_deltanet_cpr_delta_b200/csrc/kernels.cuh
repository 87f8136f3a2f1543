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
// Position-sensitive hash of cu_seqlens: the wrapping sum over n of
// mix64((n << 32) | cu[n]) (the splitmix64 finalizer).  The host computes the
// same sum from its copy; the device recomputes it from the device copy.
__host__ __device__ inline uint64_t cu_entry_hash(int n, int32_t value)
{
    uint64_t z = ((uint64_t)(uint32_t)n << 32) | (uint64_t)(uint32_t)value;
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// One CTA.  For every sequence n (L_n = cu[n+1]-cu[n]):
//   cto[n] = sum_{m<n} ceil(L_m/C)      (chunk tasks of k_tok)
//   fco[n] = sum_{m<n} floor(L_m/C)     (full chunks: k_prep / k_chain)
//   so[n]  = sum_{m<n} (floor(L_m/C)+1) (chunk-state slots)
// and the totals at index N.  err[0] = 1 if the device cu_seqlens is invalid
// or disagrees with the host copy (totals or hash); every later kernel then
// exits without writing.
__global__ void k_tables(const int32_t* __restrict__ cu, int N, int C, int64_t T_total,
                         int64_t want_tasks, int64_t want_full, int64_t want_states, uint64_t want_hash,
                         int32_t* cto, int32_t* fco, int32_t* so, int32_t* err)
{
    __shared__ long long wsum[3][32];
    __shared__ long long tot[3];
    __shared__ unsigned long long hsum;
    __shared__ int bad_any;
    const int tid = threadIdx.x, nth = blockDim.x;
    if (tid == 0) { bad_any = 0; hsum = 0ull; }
    __syncthreads();
    const int per = (N + nth - 1) / nth;
    const int n0 = min(N, tid * per), n1 = min(N, n0 + per);
    long long a = 0, b = 0, c = 0;
    unsigned long long hs = 0ull;
    int bad = 0;
    for (int n = n0; n < n1; ++n) {
        const int L = cu[n + 1] - cu[n];
        if (L < 0) bad = 1;
        const int Lc = L < 0 ? 0 : L;
        a += (Lc + C - 1) / C;
        b += Lc / C;
        c += Lc / C + 1;
        hs += cu_entry_hash(n, cu[n]);
    }
    if (tid == 0) hs += cu_entry_hash(N, cu[N]);
    atomicAdd(&hsum, hs);
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
                        tot[0] == want_tasks && tot[1] == want_full && tot[2] == want_states &&
                        hsum == want_hash;
        err[0] = ok ? 0 : 1;
    }
}
// ------------------------------------------------------------------ P_tok
// Per-thread share of one state row in the P_tok kernels: 4 consecutive lanes
// own a row, lane p holds elements [p*EPT, (p+1)*EPT), which are leaves 2p
// and 2p+1.  The two leaves' chains are independent, so they run packed:
// register pair m holds (leaf 2p element m, leaf 2p+1 element m).
template <int DK>
struct RowSplit {
    static constexpr int TPR = 4;
    static constexpr int EPT = DK / TPR;      // elements per lane
    static constexpr int L = DK / kLeaves;    // leaf length = packed pairs per lane
    static constexpr int PAD = EPT >= 16 ? 4 : 0;
    static constexpr int PS = EPT + PAD;      // smem stride between the lanes' slices
    static constexpr int KS = TPR * PS;       // smem row stride (floats)
    static_assert(L % 2 == 0, "pairs are read 16 bytes at a time");
    // smem slot of element j: slices of the 4 lanes, each holding its two
    // leaves interleaved, so one 16-byte read yields two packed pairs.  PAD
    // keeps the 4 lanes' reads in distinct banks.
    __host__ __device__ static constexpr int slot(int j)
    {
        return (j / EPT) * PS + ((j % EPT) < L ? 2 * (j % EPT) : 2 * (j % EPT - L) + 1);
    }
};

// One P_tok step on this lane's share of a row.  kt/qt point at this lane's
// slice of k_t/q_t in smem (slot layout).  Returns o_t[row] (the same bits in
// all 4 lanes of the row).
template <int DK>
__device__ __forceinline__ float ptok_step(f2x (&Rp)[DK / kLeaves], const float* kt, const float* qt, float v_i,
                                           float a, float b)
{
    constexpr int L = DK / kLeaves;
    f2x kp[L];
#pragma unroll
    for (int m = 0; m < L; m += 2) {
        const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(kt + 2 * m);
        kp[m] = x.x;
        kp[m + 1] = x.y;
    }
    f2x acc = fmul2(Rp[0], kp[0]);
#pragma unroll
    for (int m = 1; m < L; ++m) acc = ffma2(Rp[m], kp[m], acc);
    float la, lb;
    up2(acc, la, lb);
    const float u = tree_4lanes(la, lb);
    const float d = fmul(b, fsub(v_i, fmul(a, u)));
    const f2x aa = pk2(a, a), dd = pk2(d, d);
#pragma unroll
    for (int m = 0; m < L; ++m) Rp[m] = ffma2(dd, kp[m], fmul2(aa, Rp[m]));
    f2x qp[L];
#pragma unroll
    for (int m = 0; m < L; m += 2) {
        const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(qt + 2 * m);
        qp[m] = x.x;
        qp[m + 1] = x.y;
    }
    acc = fmul2(Rp[0], qp[0]);
#pragma unroll
    for (int m = 1; m < L; ++m) acc = ffma2(Rp[m], qp[m], acc);
    up2(acc, la, lb);
    return tree_4lanes(la, lb);
}

// This lane's slice of a state row (global, EPT contiguous floats) -> packed pairs.
template <int DK>
__device__ __forceinline__ void load_row_pairs(f2x (&Rp)[DK / kLeaves], const float* src)
{
    using RS = RowSplit<DK>;
    float t[RS::EPT];
#pragma unroll
    for (int e = 0; e < RS::EPT; e += 4) {
        const float4 x = *reinterpret_cast<const float4*>(src + e);
        t[e] = x.x; t[e + 1] = x.y; t[e + 2] = x.z; t[e + 3] = x.w;
    }
#pragma unroll
    for (int m = 0; m < RS::L; ++m) Rp[m] = pk2(t[m], t[RS::L + m]);
}

template <int DK>
__device__ __forceinline__ void store_row_pairs(float* dst, const f2x (&Rp)[DK / kLeaves])
{
    using RS = RowSplit<DK>;
    float t[RS::EPT];
#pragma unroll
    for (int m = 0; m < RS::L; ++m) up2(Rp[m], t[m], t[RS::L + m]);
#pragma unroll
    for (int e = 0; e < RS::EPT; e += 4)
        *reinterpret_cast<float4*>(dst + e) = make_float4(t[e], t[e + 1], t[e + 2], t[e + 3]);
}

// Stage `len` tokens of a [T,H,D] input (rows tok0.., head h) into smem rows
// of stride `ld`, widened to fp32; element j goes to column idx(j).
template <int D, typename IdxFn>
__device__ __forceinline__ void stage_rows(float* dst, int ld, const void* src, int64_t tok0, int len, int H,
                                           int h, int bf16, IdxFn idx)
{
    for (int e = threadIdx.x; e < len * (D / 8); e += blockDim.x) {
        const int t = e / (D / 8), j8 = (e % (D / 8)) * 8;
        float x[8];
        load8(src, ((tok0 + t) * H + h) * (int64_t)D + j8, bf16, x);
        float* d = dst + t * ld;
#pragma unroll
        for (int m = 0; m < 8; ++m) d[idx(j8 + m)] = x[m];
    }
}

struct IdxIdentity {
    __device__ int operator()(int j) const { return j; }
};
template <int DK>
struct IdxSlot {
    __device__ int operator()(int j) const { return RowSplit<DK>::slot(j); }
};

// P_tok on RHO rows at once: every k/q pair read from smem serves RHO rows,
// which cuts shared-memory traffic per flop by RHO.  Rp[r] is row r's share;
// v[r] its value-channel input; returns o in o[r].
template <int DK, int RHO>
__device__ __forceinline__ void ptok_rows(f2x (&Rp)[RHO][DK / kLeaves], const float* kt, const float* qt,
                                          const float (&v)[RHO], float a, float b, float (&o)[RHO])
{
    constexpr int L = DK / kLeaves;
    f2x kp[L];
#pragma unroll
    for (int m = 0; m < L; m += 2) {
        const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(kt + 2 * m);
        kp[m] = x.x;
        kp[m + 1] = x.y;
    }
    f2x acc[RHO];
#pragma unroll
    for (int r = 0; r < RHO; ++r) acc[r] = fmul2(Rp[r][0], kp[0]);
#pragma unroll
    for (int m = 1; m < L; ++m)
#pragma unroll
        for (int r = 0; r < RHO; ++r) acc[r] = ffma2(Rp[r][m], kp[m], acc[r]);
    const f2x aa = pk2(a, a);
    f2x dd[RHO];
#pragma unroll
    for (int r = 0; r < RHO; ++r) {
        float la, lb;
        up2(acc[r], la, lb);
        const float u = tree_4lanes(la, lb);
        const float d = fmul(b, fsub(v[r], fmul(a, u)));
        dd[r] = pk2(d, d);
    }
#pragma unroll
    for (int m = 0; m < L; ++m)
#pragma unroll
        for (int r = 0; r < RHO; ++r) Rp[r][m] = ffma2(dd[r], kp[m], fmul2(aa, Rp[r][m]));
#pragma unroll
    for (int m = 0; m < L; m += 2) {
        const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(qt + 2 * m);
        kp[m] = x.x;
        kp[m + 1] = x.y;
    }
#pragma unroll
    for (int r = 0; r < RHO; ++r) acc[r] = fmul2(Rp[r][0], kp[0]);
#pragma unroll
    for (int m = 1; m < L; ++m)
#pragma unroll
        for (int r = 0; r < RHO; ++r) acc[r] = ffma2(Rp[r][m], kp[m], acc[r]);
#pragma unroll
    for (int r = 0; r < RHO; ++r) {
        float la, lb;
        up2(acc[r], la, lb);
        o[r] = tree_4lanes(la, lb);
    }
}

// k_tok layout: one CTA per (chunk task, head) covers all DV rows; lane
// (g, p) owns rows RHO*g .. RHO*g+RHO-1, share p.  The chunk's k, q, v and
// gates are staged SC tokens at a time: raw bytes arrive by cp.async while
// the previous sub-chunk computes, then are widened into the fp32 buffers.
template <int DK, int DV, int C>
struct TokCfg {
    using RS = RowSplit<DK>;
    static constexpr int RHO = DV >= 32 ? 4 : 2;          // rows per lane
    static constexpr int THREADS = (DV / RHO) * RS::TPR;   // >= 32
    static constexpr int SC = 16;                          // tokens per sub-chunk
    static constexpr int RAW_TOK = (2 * DK + DV) * 4;      // raw bytes per token (fp32 inputs; bf16 uses half)
    static constexpr int KQ_OFF = 0;                       // floats: [SC][2][KS]
    static constexpr int VS_OFF = KQ_OFF + SC * 2 * RS::KS;  // [SC][DV]
    static constexpr int OS_OFF = VS_OFF + SC * DV;          // [SC][DV]
    static constexpr int AB_OFF = OS_OFF + SC * DV;          // [2][SC]
    static constexpr int RAB_OFF = AB_OFF + 2 * SC;          // raw gates [2][SC]
    static constexpr int RAW_OFF = RAB_OFF + 2 * SC;         // raw token bytes [SC][RAW_TOK]
    static constexpr size_t SMEM = sizeof(float) * RAW_OFF + (size_t)SC * RAW_TOK;
    static_assert(THREADS % 32 == 0, "whole warps (the tree shuffles use full masks)");
};

// 8 consecutive elements of a raw bf16/fp32 token row in smem, widened to fp32.
__device__ __forceinline__ void lds8_raw(const unsigned char* base, int el, int bf16, float* o)
{
    if (bf16) {
        const uint4 u = *reinterpret_cast<const uint4*>(base + 2 * el);
        o[0] = __uint_as_float(u.x << 16); o[1] = __uint_as_float(u.x & 0xffff0000u);
        o[2] = __uint_as_float(u.y << 16); o[3] = __uint_as_float(u.y & 0xffff0000u);
        o[4] = __uint_as_float(u.z << 16); o[5] = __uint_as_float(u.z & 0xffff0000u);
        o[6] = __uint_as_float(u.w << 16); o[7] = __uint_as_float(u.w & 0xffff0000u);
    } else {
        const float4 a = *reinterpret_cast<const float4*>(base + 4 * el);
        const float4 b = *reinterpret_cast<const float4*>(base + 4 * el + 16);
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
        o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
    }
}

// Intra-chunk recurrence: one CTA per (chunk task, head).
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
    constexpr int RHO = Cf::RHO, SC = Cf::SC, L = RS::L, KS = RS::KS;
    if (__ldg(err)) return;
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    float* kq = sm + Cf::KQ_OFF;
    float* vs = sm + Cf::VS_OFF;
    float* os = sm + Cf::OS_OFF;
    float* ab = sm + Cf::AB_OFF;
    float* rab = sm + Cf::RAB_OFF;
    unsigned char* raw = reinterpret_cast<unsigned char*>(sm + Cf::RAW_OFF);

    const int h = blockIdx.x % H;
    const int g = blockIdx.x / H;
    const int n = find_seq(cto, N, g);
    const int c = g - __ldg(cto + n);
    const int seq0 = __ldg(cu + n);
    const int Ln = __ldg(cu + n + 1) - seq0;
    const int64_t tok0 = (int64_t)seq0 + (int64_t)c * C;
    const int len = min(C, Ln - c * C);
    const int64_t slot = (int64_t)__ldg(so + n) + c;
    const int esz = in_bf16 ? 2 : 4;
    const int kb = DK * esz, vb = DV * esz, tb = 2 * kb + vb;  // bytes per k/q row, v row, token

    // async copies of sub-chunk s: raw token rows [k | q | v] and the gates
    auto fetch = [&](int s) {
        const int t0 = s * SC, ls = min(SC, len - t0), pieces = tb / 16;
        for (int e = threadIdx.x; e < ls * pieces; e += blockDim.x) {
            const int t = e / pieces, off = (e % pieces) * 16;
            const int64_t row = (tok0 + t0 + t) * H + h;
            const char* src = off < kb ? reinterpret_cast<const char*>(k) + row * kb + off
                            : off < 2 * kb ? reinterpret_cast<const char*>(q) + row * kb + (off - kb)
                                           : reinterpret_cast<const char*>(v) + row * vb + (off - 2 * kb);
            cp_async16(raw + t * Cf::RAW_TOK + off, src);
        }
        for (int t = threadIdx.x; t < ls; t += blockDim.x) {
            cp_async4(rab + t, alpha + (tok0 + t0 + t) * H + h);
            cp_async4(rab + SC + t, beta + (tok0 + t0 + t) * H + h);
        }
        cp_async_commit();
    };
    // raw sub-chunk -> fp32: k, q in the slot layout, v by row, gates
    auto widen = [&](int ls) {
        constexpr int G8 = (2 * DK + DV) / 8;
        for (int e = threadIdx.x; e < ls * G8; e += blockDim.x) {
            const int t = e / G8, el = (e % G8) * 8;
            float x[8];
            lds8_raw(raw + t * Cf::RAW_TOK, el, in_bf16, x);
            if (el < 2 * DK) {
                float* d = kq + (t * 2 + (el >= DK)) * KS;
                const int j = el >= DK ? el - DK : el;
#pragma unroll
                for (int m = 0; m < 8; ++m) d[RS::slot(j + m)] = x[m];
            } else {
#pragma unroll
                for (int m = 0; m < 8; ++m) vs[t * DV + (el - 2 * DK) + m] = x[m];
            }
        }
        for (int t = threadIdx.x; t < ls; t += blockDim.x) {
            ab[t] = rab[t];
            ab[SC + t] = rab[SC + t];
        }
    };

    const int gi = threadIdx.x / RS::TPR, p = threadIdx.x % RS::TPR;
    const int row0 = gi * RHO;
    f2x Rp[RHO][L];
#pragma unroll
    for (int r = 0; r < RHO; ++r)
        load_row_pairs<DK>(Rp[r], states + ((slot * H + h) * DV + row0 + r) * DK + p * RS::EPT);

    const int nsub = (len + SC - 1) / SC;
    fetch(0);
    for (int s = 0; s < nsub; ++s) {
        const int ls = min(SC, len - s * SC);
        cp_async_wait_all();
        __syncthreads();  // raw(s) landed; the previous sub-chunk's outputs are stored
        widen(ls);
        __syncthreads();  // fp32 buffers ready; raw is free again
        if (s + 1 < nsub) fetch(s + 1);
        for (int t = 0; t < ls; ++t) {
            float vv[RHO], oo[RHO];
#pragma unroll
            for (int r = 0; r < RHO; ++r) vv[r] = vs[t * DV + row0 + r];
            ptok_rows<DK, RHO>(Rp, kq + (t * 2) * KS + p * RS::PS, kq + (t * 2 + 1) * KS + p * RS::PS, vv,
                               ab[t], ab[SC + t], oo);
            if (p == 0) {
#pragma unroll
                for (int r = 0; r < RHO; ++r) os[t * DV + row0 + r] = oo[r];
            }
        }
        __syncthreads();
        for (int e = threadIdx.x; e < ls * (DV / 8); e += blockDim.x) {
            const int t = e / (DV / 8), i8 = (e % (DV / 8)) * 8;
            store8(o, ((tok0 + s * SC + t) * H + h) * (int64_t)DV + i8, out_bf16, os + t * DV + i8);
        }
    }

    if (cacheR != nullptr && len < C) {  // last, partial chunk: the running state for decode
#pragma unroll
        for (int r = 0; r < RHO; ++r)
            store_row_pairs<DK>(cacheR + (((int64_t)n * H + h) * DV + row0 + r) * DK + p * RS::EPT, Rp[r]);
    }
}

// ------------------------------------------------------------------ P_chunk
template <int DK, int DV, int C>
struct ChunkCfg {
    static constexpr int KS = DK + 4;      // padded k / w / S row stride
    static constexpr int C1 = C + 1;       // decay matrix row stride
    static constexpr int CT = C + 4;       // c^T row stride
    static constexpr int DCS = C + 4;      // stride of D[C][.] rows in the workspace
    static constexpr int RTB = DV < 32 ? DV : 32;  // boundary-state rows per tile
    static constexpr int NTB = DV / RTB;
    static constexpr int THREADS = 256;
};

// VEC consecutive floats from smem (VEC = 4 or 2; 4*VEC-byte aligned).
template <int VEC>
__device__ __forceinline__ void lds_n(float (&r)[VEC], const float* s)
{
    if constexpr (VEC == 4) {
        const float4 x = *reinterpret_cast<const float4*>(s);
        r[0] = x.x; r[1] = x.y; r[2] = x.z; r[3] = x.w;
    } else {
        const float2 x = *reinterpret_cast<const float2*>(s);
        r[0] = x.x; r[1] = x.y;
    }
}

// tree(x_a, y_b) for an RA x RB block of row pairs, all rows of stride KS in
// smem: xa[r] = row r of the first operand, yb[c] = row c of the second.
// The leaves run in ascending j; VEC elements are read at a time.
template <int DK, int KS, int RA, int RB>
__device__ __forceinline__ void tree_block(const float* const (&xa)[RA], const float* const (&yb)[RB],
                                           float (&out)[RA][RB])
{
    constexpr int L = DK / kLeaves;
    constexpr int VEC = (L % 4 == 0) ? 4 : 2;
    TreeAcc st[RA][RB];
#pragma unroll
    for (int l = 0; l < kLeaves; ++l) {
        float acc[RA][RB];
#pragma unroll
        for (int m = 0; m < L; m += VEC) {
            float a[RA][VEC], b[RB][VEC];
#pragma unroll
            for (int r = 0; r < RA; ++r) lds_n<VEC>(a[r], xa[r] + l * L + m);
#pragma unroll
            for (int c = 0; c < RB; ++c) lds_n<VEC>(b[c], yb[c] + l * L + m);
#pragma unroll
            for (int e = 0; e < VEC; ++e)
#pragma unroll
                for (int r = 0; r < RA; ++r)
#pragma unroll
                    for (int c = 0; c < RB; ++c)
                        acc[r][c] = (m + e == 0) ? fmul(a[r][e], b[c][e]) : ffma(a[r][e], b[c][e], acc[r][c]);
        }
#pragma unroll
        for (int r = 0; r < RA; ++r)
#pragma unroll
            for (int c = 0; c < RB; ++c) tree_push(st[r][c], l, acc[r][c]);
    }
#pragma unroll
    for (int r = 0; r < RA; ++r)
#pragma unroll
        for (int c = 0; c < RB; ++c) out[r][c] = st[r][c].t0;
}

// Forward substitution of one column, right-looking and fully unrolled: once
// token s is final, its term enters every later token's chain.  For each
// token t the chain still runs over s = 1..t-1 in ascending order.
// acc[t] holds the chain start on entry and the column's result on exit.
template <int C, int CT>
__device__ __forceinline__ void fwd_subst(float (&acc)[C], const float* cT, const float* bs)
{
#pragma unroll
    for (int sig = 0; sig < C; ++sig) {
        acc[sig] = fmul(bs[sig], acc[sig]);
        const float x = acc[sig];
#pragma unroll
        for (int tg = (sig + 1) / 4; tg < C / 4; ++tg) {
            const float4 c4 = *reinterpret_cast<const float4*>(cT + sig * CT + 4 * tg);
            if (4 * tg + 0 > sig) acc[4 * tg + 0] = ffma(-c4.x, x, acc[4 * tg + 0]);
            if (4 * tg + 1 > sig) acc[4 * tg + 1] = ffma(-c4.y, x, acc[4 * tg + 1]);
            if (4 * tg + 2 > sig) acc[4 * tg + 2] = ffma(-c4.z, x, acc[4 * tg + 2]);
            if (4 * tg + 3 > sig) acc[4 * tg + 3] = ffma(-c4.w, x, acc[4 * tg + 3]);
        }
    }
}

// P_chunk part 1 for one chunk, by one CTA.  ks [C][KS], vs [C][DV], as/bs [C]
// in smem.  Dm [(C+1)^2] and cT [C][CT] are smem scratch.  Writes
//   w_t  -> wout[(t-1)*ldw + j],   u0_t -> uout[(t-1)*ldu + i],   D[C][s] -> dCout[s]
// (any address space).  uout may alias vs: each column of vs is read only by
// the thread that later writes that column of uout, and only before it does.
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
    // c[t][s] = D[t][s] * tree(k_s, k_t), stored transposed: cT[s-1][t-1];
    // 4x4 blocks of the strictly lower triangle, one block per thread
    constexpr int NB = C / 4, NBLK = NB * (NB + 1) / 2;
    for (int blk = threadIdx.x; blk < NBLK; blk += blockDim.x) {
        int bt = 0;
        while ((bt + 1) * (bt + 2) / 2 <= blk) ++bt;
        const int bsg = blk - bt * (bt + 1) / 2;
        const float* const xa[4] = {ks + (4 * bt) * KS, ks + (4 * bt + 1) * KS, ks + (4 * bt + 2) * KS,
                                    ks + (4 * bt + 3) * KS};
        const float* const yb[4] = {ks + (4 * bsg) * KS, ks + (4 * bsg + 1) * KS, ks + (4 * bsg + 2) * KS,
                                    ks + (4 * bsg + 3) * KS};
        float G[4][4];
        tree_block<DK, KS, 4, 4>(xa, yb, G);
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int tau = 4 * bt + r, sig = 4 * bsg + c;
                if (sig < tau) cT[sig * CT + tau] = fmul(Dm[(tau + 1) * C1 + (sig + 1)], G[r][c]);
            }
    }
    if (dCout != nullptr)
        for (int s = threadIdx.x; s <= C; s += blockDim.x) dCout[s] = Dm[C * C1 + s];
    __syncthreads();
    // forward substitution, one column per thread
    for (int col = threadIdx.x; col < DV + DK; col += blockDim.x) {
        float acc[C];
        if (col < DV) {
#pragma unroll
            for (int tau = 0; tau < C; ++tau) acc[tau] = vs[tau * DV + col];
            fwd_subst<C, CT>(acc, cT, bs);
#pragma unroll
            for (int tau = 0; tau < C; ++tau) uout[tau * ldu + col] = acc[tau];
        } else {
            const int j = col - DV;
#pragma unroll
            for (int tau = 0; tau < C; ++tau) acc[tau] = fmul(Dm[(tau + 1) * C1], ks[tau * KS + j]);
            fwd_subst<C, CT>(acc, cT, bs);
#pragma unroll
            for (int tau = 0; tau < C; ++tau) wout[tau * ldw + j] = acc[tau];
        }
    }
    __syncthreads();
}

// P_chunk part 2 on a tile of RTB boundary-state rows, by one CTA:
//   e_t[i] = D[C][t] * (u0_t[i] - tree(S_i, w_t)),
//   S_ij <- chain_t fma(e_t[i], k_t[j], .) from D[C][0] * S_ij.
// Ss [RTB][KS], ws [C][KS], ks [C][KS], us [C][ldu], dCs [C+1], es [C][RTB]
// (scratch), all smem.  The new rows also go to dst1 / dst2 (global, row
// stride DK) when non-null.
template <int DK, int RTB, int C>
__device__ __forceinline__ void chunk_advance(float* Ss, const float* ws, const float* us, int ldu,
                                              const float* ks, const float* dCs, float* es, float* dst1,
                                              float* dst2)
{
    constexpr int KS = DK + 4;
    // phase 1: tiles of 4 tokens x 2 rows (rows ig and ig + RTB/2)
    constexpr int IG = RTB / 2, TG = C / 4;
    for (int tile = threadIdx.x; tile < TG * IG; tile += blockDim.x) {
        const int ig = tile % IG, tg = tile / IG;
        const float* const xa[4] = {ws + (4 * tg) * KS, ws + (4 * tg + 1) * KS, ws + (4 * tg + 2) * KS,
                                    ws + (4 * tg + 3) * KS};
        const float* const yb[2] = {Ss + ig * KS, Ss + (ig + IG) * KS};
        float sw[4][2];
        tree_block<DK, KS, 4, 2>(xa, yb, sw);
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int tau = 4 * tg + r, i = ig + c * IG;
                es[tau * RTB + i] = fmul(dCs[tau + 1], fsub(us[tau * ldu + i], sw[r][c]));
            }
    }
    __syncthreads();
    // phase 2: tiles of 4 rows x 4 columns
    constexpr int JG = DK / 4, IG2 = RTB / 4;
    const float d0 = dCs[0];
    for (int tile = threadIdx.x; tile < IG2 * JG; tile += blockDim.x) {
        const int jg = tile % JG, ig = tile / JG;
        float acc[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const float4 s = *reinterpret_cast<const float4*>(Ss + (4 * ig + r) * KS + 4 * jg);
            acc[r][0] = fmul(d0, s.x); acc[r][1] = fmul(d0, s.y);
            acc[r][2] = fmul(d0, s.z); acc[r][3] = fmul(d0, s.w);
        }
#pragma unroll 4
        for (int tau = 0; tau < C; ++tau) {
            const float4 e4 = *reinterpret_cast<const float4*>(es + tau * RTB + 4 * ig);
            const float4 k4 = *reinterpret_cast<const float4*>(ks + tau * KS + 4 * jg);
            const float ev[4] = {e4.x, e4.y, e4.z, e4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[r][c] = ffma(ev[r], kv[c], acc[r][c]);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const float4 x = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
            *reinterpret_cast<float4*>(Ss + (4 * ig + r) * KS + 4 * jg) = x;  // element owned by this thread
            if (dst1 != nullptr) *reinterpret_cast<float4*>(dst1 + (int64_t)(4 * ig + r) * DK + 4 * jg) = x;
            if (dst2 != nullptr) *reinterpret_cast<float4*>(dst2 + (int64_t)(4 * ig + r) * DK + 4 * jg) = x;
        }
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
        for (int e = threadIdx.x; e < C * (RTB / 4); e += blockDim.x) {
            const int t = e / (RTB / 4), i4 = (e % (RTB / 4)) * 4;
            *reinterpret_cast<float4*>(us + t * RTB + i4) = __ldg(reinterpret_cast<const float4*>(usrc + t * DV + i4));
        }
        for (int s = threadIdx.x; s <= C; s += blockDim.x) dCs[s] = __ldg(dC_ws + task * Cf::DCS + s);
        __syncthreads();
        chunk_advance<DK, RTB, C>(Ss, ws, us, RTB, ks, dCs, es,
                                  states + (((slot0 + c + 1) * H + h) * DV + row0) * DK, nullptr);
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
    static constexpr int RT = DV < 32 ? DV : 32;  // rows per CTA
    static constexpr int NT = DV / RT;
    static constexpr int THREADS = RT * RS::TPR;
};

// One decode token per (sequence, head), one CTA per row tile: P_tok on the
// running state R; tile 0 also appends the token to the buffer at slot pos.
// pos itself is advanced by k_dec_resync, which runs next.
template <int DK, int DV, int C>
__global__ void __launch_bounds__(DecCfg<DK, DV>::THREADS)
k_dec_tok(const void* __restrict__ q, const void* __restrict__ k, const void* __restrict__ v,
          const float* __restrict__ alpha, const float* __restrict__ beta, int in_bf16, int out_bf16,
          float* R, void* kbuf, void* vbuf, float* abuf, float* bbuf, const int32_t* pos, void* __restrict__ o)
{
    using Cf = DecCfg<DK, DV>;
    using RS = typename Cf::RS;
    __shared__ __align__(16) float ks[RS::KS];
    __shared__ __align__(16) float qs[RS::KS];
    __shared__ __align__(16) float vs[Cf::RT];
    const int nh = blockIdx.x / Cf::NT, r = blockIdx.x % Cf::NT;
    const int p = pos[nh];
    if (p < 0 || p >= C) return;
    stage_rows<DK>(ks, RS::KS, k, nh, 1, 1, 0, in_bf16, IdxSlot<DK>());
    stage_rows<DK>(qs, RS::KS, q, nh, 1, 1, 0, in_bf16, IdxSlot<DK>());
    for (int e = threadIdx.x; e < Cf::RT / 8; e += blockDim.x) {
        float x[8];
        load8(v, (int64_t)nh * DV + r * Cf::RT + e * 8, in_bf16, x);
#pragma unroll
        for (int m = 0; m < 8; ++m) vs[e * 8 + m] = x[m];
    }
    const float a = __ldg(alpha + nh), b = __ldg(beta + nh);
    const int row = threadIdx.x / RS::TPR, part = threadIdx.x % RS::TPR;
    const int grow = r * Cf::RT + row;
    float* Rrow = R + ((int64_t)nh * DV + grow) * DK + part * RS::EPT;
    f2x Rp[RS::L];
    load_row_pairs<DK>(Rp, Rrow);
    __syncthreads();
    const float ot = ptok_step<DK>(Rp, ks + part * RS::PS, qs + part * RS::PS, vs[row], a, b);
    store_row_pairs<DK>(Rrow, Rp);
    if (part == 0) store1(o, (int64_t)nh * DV + grow, out_bf16, ot);
    if (r == 0) {  // append the raw token to the buffer at slot p
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
    }
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

// Advances pos after k_dec_tok appended a token at slot pos, and resyncs
// where that token completed a chunk: S_b <- P_chunk(S_b, buffer), R <- S_b,
// pos <- 0.  Persistent: CTA b handles (sequence, head) pairs b, b + grid, ...
// A pos outside [0, C) is left unchanged.
template <int DK, int DV, int C>
__global__ void __launch_bounds__(256)
k_dec_resync(int NH, int in_bf16, float* S_b, float* R, const void* kbuf, const void* vbuf, const float* abuf,
             const float* bbuf, int32_t* pos)
{
    using Cf = ChunkCfg<DK, DV, C>;
    using Sm = ResyncSmem<DK, DV, C>;
    constexpr int KS = Cf::KS, RTB = Cf::RTB;
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

    for (int nh = blockIdx.x; nh < NH; nh += gridDim.x) {
        const int p = pos[nh];
        __syncthreads();  // every thread has read pos (and the previous pair's smem) before anything moves
        if (p < 0 || p >= C) continue;
        if (p + 1 < C) {
            if (threadIdx.x == 0) pos[nh] = p + 1;
            continue;
        }
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
            chunk_advance<DK, RTB, C>(Ss, ws, vs + r * RTB, DV, ks, dCs, es, Sg, Rg);
        }
        if (threadIdx.x == 0) pos[nh] = 0;
    }
}

}  // namespace gdn
