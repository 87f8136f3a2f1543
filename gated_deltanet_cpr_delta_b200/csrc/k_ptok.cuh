// k_ptok.cuh -- per-token recurrence P_tok and the intra-chunk kernel k_tok (sm_100a).
#pragma once

#include "schedule.cuh"

namespace gdn {

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

// Barriers for a P_tok task: the whole CTA, or one 128-thread half of a
// larger CTA (named barrier `id`).
struct CtaSync {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};
struct HalfSync {
    int id;
    __device__ __forceinline__ void operator()() const { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }
};

// Intra-chunk recurrence for chunk c of sequence n (tokens seq0 + cC ..), head
// h, by TokCfg::THREADS threads (tid = 0..THREADS-1) with smem `sm` of
// TokCfg::SMEM bytes.  The chunk starts from states[slot] (COHERENT: read
// through L2, for states written earlier in the same launch).
template <int DK, int DV, int C, bool COHERENT, typename Sync>
__device__ __forceinline__ void tok_task(const void* __restrict__ q, const void* __restrict__ k,
                                         const void* __restrict__ v, const float* __restrict__ alpha,
                                         const float* __restrict__ beta, int n, int c, int h, int H, int seq0, int Ln,
                                         int64_t slot, int in_bf16, int out_bf16, const float* states,
                                         void* __restrict__ o, float* __restrict__ cacheR, float* sm, int tid,
                                         Sync sync)
{
    using Cf = TokCfg<DK, DV, C>;
    using RS = typename Cf::RS;
    constexpr int RHO = Cf::RHO, SC = Cf::SC, L = RS::L, KS = RS::KS, NT = Cf::THREADS;
    float* kq = sm + Cf::KQ_OFF;
    float* vs = sm + Cf::VS_OFF;
    float* os = sm + Cf::OS_OFF;
    float* ab = sm + Cf::AB_OFF;
    float* rab = sm + Cf::RAB_OFF;
    unsigned char* raw = reinterpret_cast<unsigned char*>(sm + Cf::RAW_OFF);

    const int64_t tok0 = (int64_t)seq0 + (int64_t)c * C;
    const int len = min(C, Ln - c * C);
    const int esz = in_bf16 ? 2 : 4;
    const int kb = DK * esz, vb = DV * esz, tb = 2 * kb + vb;  // bytes per k/q row, v row, token

    // async copies of sub-chunk s: raw token rows [k | q | v] and the gates
    auto fetch = [&](int s) {
        const int t0 = s * SC, ls = min(SC, len - t0), pieces = tb / 16;
        for (int e = tid; e < ls * pieces; e += NT) {
            const int t = e / pieces, off = (e % pieces) * 16;
            const int64_t row = (tok0 + t0 + t) * H + h;
            const char* src = off < kb ? reinterpret_cast<const char*>(k) + row * kb + off
                            : off < 2 * kb ? reinterpret_cast<const char*>(q) + row * kb + (off - kb)
                                           : reinterpret_cast<const char*>(v) + row * vb + (off - 2 * kb);
            cp_async16(raw + t * Cf::RAW_TOK + off, src);
        }
        for (int t = tid; t < ls; t += NT) {
            cp_async4(rab + t, alpha + (tok0 + t0 + t) * H + h);
            cp_async4(rab + SC + t, beta + (tok0 + t0 + t) * H + h);
        }
        cp_async_commit();
    };
    // raw sub-chunk -> fp32: k, q in the slot layout, v by row, gates
    auto widen = [&](int ls) {
        constexpr int G8 = (2 * DK + DV) / 8;
        for (int e = tid; e < ls * G8; e += NT) {
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
        for (int t = tid; t < ls; t += NT) {
            ab[t] = rab[t];
            ab[SC + t] = rab[SC + t];
        }
    };

    const int gi = tid / RS::TPR, p = tid % RS::TPR;
    const int row0 = gi * RHO;
    f2x Rp[RHO][L];
#pragma unroll
    for (int r = 0; r < RHO; ++r) {
        const float* src = states + ((slot * H + h) * DV + row0 + r) * DK + p * RS::EPT;
        if (COHERENT) {
            float t[RS::EPT];
#pragma unroll
            for (int e = 0; e < RS::EPT; e += 4) {
                const float4 x = __ldcg(reinterpret_cast<const float4*>(src + e));
                t[e] = x.x; t[e + 1] = x.y; t[e + 2] = x.z; t[e + 3] = x.w;
            }
#pragma unroll
            for (int m = 0; m < L; ++m) Rp[r][m] = pk2(t[m], t[L + m]);
        } else {
            load_row_pairs<DK>(Rp[r], src);
        }
    }

    const int nsub = (len + SC - 1) / SC;
    fetch(0);
    for (int s = 0; s < nsub; ++s) {
        const int ls = min(SC, len - s * SC);
        cp_async_wait_all();
        sync();  // raw(s) landed; the previous sub-chunk's outputs are stored
        widen(ls);
        sync();  // fp32 buffers ready; raw is free again
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
        sync();
        for (int e = tid; e < ls * (DV / 8); e += NT) {
            const int t = e / (DV / 8), i8 = (e % (DV / 8)) * 8;
            store8(o, ((tok0 + s * SC + t) * H + h) * (int64_t)DV + i8, out_bf16, os + t * DV + i8);
        }
    }

    if (cacheR != nullptr && len < C) {  // last, partial chunk: the running state for decode
#pragma unroll
        for (int r = 0; r < RHO; ++r)
            store_row_pairs<DK>(cacheR + (((int64_t)n * H + h) * DV + row0 + r) * DK + p * RS::EPT, Rp[r]);
    }
    sync();  // smem free for the next task
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
    if (__ldg(err)) return;
    extern __shared__ float4 smem_f4[];
    const int h = blockIdx.x % H;
    const int g = blockIdx.x / H;
    const int n = find_seq(cto, N, g);
    const int c = g - __ldg(cto + n);
    const int seq0 = __ldg(cu + n);
    tok_task<DK, DV, C, false>(q, k, v, alpha, beta, n, c, h, H, seq0, __ldg(cu + n + 1) - seq0,
                               (int64_t)__ldg(so + n) + c, in_bf16, out_bf16, states, o, cacheR,
                               reinterpret_cast<float*>(smem_f4), threadIdx.x, CtaSync{});
}

}  // namespace gdn
