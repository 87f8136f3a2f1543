// k_ptok.cuh -- per-token recurrence P_tok and the intra-chunk kernel k_tok (sm_100a).
#pragma once

#include "schedule.cuh"
#include "tma.cuh"

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

// The running state of P_tok is kept scaled: the state is c * Rt, with a
// scalar c per (sequence, head) and Rt the d_v x d_k matrix the kernels hold.
// The decay alpha_t then multiplies c instead of every element.  When the new
// scale alpha_t * c would fall below kFoldTau, it is folded into Rt instead
// (Rt <- (alpha_t c) Rt, c <- 1), which keeps Rt = state / c within 2^64 of the
// state's own magnitude and handles alpha_t = 0 (a reset) exactly.
constexpr float kFoldTau = 0x1p-64f;

// The scalars of one token for one row, from the dots over Rt before the token:
//   cn = alpha * c;  d = beta * (v - cn * dk)
//   no fold (cn >= tau): dt = d * rcp(cn),  o = cn * fma(dt, kq, dq)
//   fold:                dt = d,            o = fma(d, kq, cn * dq)
// rc = rcp(cn) (correctly rounded), or 1 for a fold.  Returns dt.
__device__ __forceinline__ float tok_scalars(float dk, float dq, float v, float b, float kq, float cn, float rc,
                                             bool fold, float& o)
{
    const float d = fmul(b, fsub(v, fmul(cn, dk)));
    if (!fold) {
        const float dt = fmul(d, rc);
        o = fmul(cn, ffma(dt, kq, dq));
        return dt;
    }
    o = ffma(d, kq, fmul(cn, dq));
    return d;
}

// Dots of RHO rows (this lane's packed share) with x and y (slot-layout slices
// in smem): the leaf chains of tree(Rt_i, x) and tree(Rt_i, y).
template <int DK, int RHO>
__device__ __forceinline__ void tok_dots(const f2x (&R)[RHO][DK / kLeaves], const float* xt, const float* yt,
                                         f2x (&ax)[RHO], f2x (&ay)[RHO])
{
    constexpr int L = DK / kLeaves;
#pragma unroll
    for (int m = 0; m < L; m += 2) {
        const ulonglong2 xx = *reinterpret_cast<const ulonglong2*>(xt + 2 * m);
        const ulonglong2 yy = *reinterpret_cast<const ulonglong2*>(yt + 2 * m);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const f2x xv = h ? xx.y : xx.x, yv = h ? yy.y : yy.x;
#pragma unroll
            for (int r = 0; r < RHO; ++r) {
                if (m + h == 0) {
                    ax[r] = fmul2(R[r][0], xv);
                    ay[r] = fmul2(R[r][0], yv);
                } else {
                    ax[r] = ffma2(R[r][m + h], xv, ax[r]);
                    ay[r] = ffma2(R[r][m + h], yv, ay[r]);
                }
            }
        }
    }
}

// Rt_i += dd_i k^T, then the dots of the new Rt with x and y (the next token's
// k and q), in one pass over the state.
template <int DK, int RHO>
__device__ __forceinline__ void tok_update_dots(f2x (&R)[RHO][DK / kLeaves], const f2x (&dd)[RHO], const float* kt,
                                                const float* xt, const float* yt, f2x (&ax)[RHO], f2x (&ay)[RHO])
{
    constexpr int L = DK / kLeaves;
#pragma unroll
    for (int m = 0; m < L; m += 2) {
        const ulonglong2 kk = *reinterpret_cast<const ulonglong2*>(kt + 2 * m);
        const ulonglong2 xx = *reinterpret_cast<const ulonglong2*>(xt + 2 * m);
        const ulonglong2 yy = *reinterpret_cast<const ulonglong2*>(yt + 2 * m);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const f2x kv = h ? kk.y : kk.x, xv = h ? xx.y : xx.x, yv = h ? yy.y : yy.x;
#pragma unroll
            for (int r = 0; r < RHO; ++r) {
                R[r][m + h] = ffma2(dd[r], kv, R[r][m + h]);
                if (m + h == 0) {
                    ax[r] = fmul2(R[r][0], xv);
                    ay[r] = fmul2(R[r][0], yv);
                } else {
                    ax[r] = ffma2(R[r][m + h], xv, ax[r]);
                    ay[r] = ffma2(R[r][m + h], yv, ay[r]);
                }
            }
        }
    }
}

template <int DK, int RHO>
__device__ __forceinline__ void tok_update(f2x (&R)[RHO][DK / kLeaves], const f2x (&dd)[RHO], const float* kt)
{
    constexpr int L = DK / kLeaves;
#pragma unroll
    for (int m = 0; m < L; m += 2) {
        const ulonglong2 kk = *reinterpret_cast<const ulonglong2*>(kt + 2 * m);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const f2x kv = h ? kk.y : kk.x;
#pragma unroll
            for (int r = 0; r < RHO; ++r) R[r][m + h] = ffma2(dd[r], kv, R[r][m + h]);
        }
    }
}

// A fold: Rt <- s * Rt.
template <int DK, int RHO>
__device__ __forceinline__ void tok_scale(f2x (&R)[RHO][DK / kLeaves], float s)
{
    constexpr int L = DK / kLeaves;
    const f2x ss = pk2(s, s);
#pragma unroll
    for (int m = 0; m < L; ++m)
#pragma unroll
        for (int r = 0; r < RHO; ++r) R[r][m] = fmul2(ss, R[r][m]);
}

// This lane's slice of a state row (EPT contiguous floats) -> packed pairs.
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

// One token of P_tok for one row on this lane's share (the decode step), with
// the token's k, q in smem (slot layout, this lane's slices) and kq = tree(k, q).
// Returns o (the same bits in the 4 lanes of the row).
template <int DK>
__device__ __forceinline__ float tok_step_row(f2x (&Rp)[DK / kLeaves], const float* kt, const float* qt, float v,
                                              float b, float kq, float cn, float rc, bool fold)
{
    f2x R1[1][DK / kLeaves];
#pragma unroll
    for (int m = 0; m < DK / kLeaves; ++m) R1[0][m] = Rp[m];
    f2x ax[1], ay[1];
    tok_dots<DK, 1>(R1, kt, qt, ax, ay);
    float la, lb;
    up2(ax[0], la, lb);
    const float dk = tree_4lanes(la, lb);
    up2(ay[0], la, lb);
    const float dq = tree_4lanes(la, lb);
    float o;
    const float dt = tok_scalars(dk, dq, v, b, kq, cn, rc, fold, o);
    if (fold) tok_scale<DK, 1>(R1, cn);
    const f2x dd[1] = {pk2(dt, dt)};
    tok_update<DK, 1>(R1, dd, kt);
#pragma unroll
    for (int m = 0; m < DK / kLeaves; ++m) Rp[m] = R1[0][m];
    return o;
}

// tree(k, q) of one token by the 4 lanes of a row group (slot-layout slices).
template <int DK>
__device__ __forceinline__ float tok_kq(const float* kt, const float* qt)
{
    constexpr int L = DK / kLeaves;
    f2x acc = 0;
#pragma unroll
    for (int m = 0; m < L; m += 2) {
        const ulonglong2 kk = *reinterpret_cast<const ulonglong2*>(kt + 2 * m);
        const ulonglong2 qq = *reinterpret_cast<const ulonglong2*>(qt + 2 * m);
        acc = m == 0 ? fmul2(kk.x, qq.x) : ffma2(kk.x, qq.x, acc);
        acc = ffma2(kk.y, qq.y, acc);
    }
    float la, lb;
    up2(acc, la, lb);
    return tree_4lanes(la, lb);
}

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

// k_tok layout: one task = (chunk, head) covers all DV rows; lane (g, p) owns
// rows RHO*g .. RHO*g+RHO-1, share p.  The chunk's k, q, v arrive SC tokens at
// a time by TMA (one box per tensor), the gates by cp.async, while the
// previous sub-chunk computes; then they are widened into the fp32 buffers.
template <int DK, int DV, int C>
struct TokCfg {
    using RS = RowSplit<DK>;
    static constexpr int RHO = DV >= 32 ? 4 : 2;           // rows per lane
    static constexpr int THREADS = (DV / RHO) * RS::TPR;   // >= 32
    static constexpr int SC = 16;                          // tokens per sub-chunk
    static constexpr int KQ_OFF = 0;                       // floats: [SC][2][KS] k, q (slot layout)
    static constexpr int VS_OFF = KQ_OFF + SC * 2 * RS::KS;  // [SC][DV]
    static constexpr int OS_OFF = VS_OFF + SC * DV;          // [SC][DV]
    static constexpr int SC_OFF = OS_OFF + SC * DV;          // [8][SC]: alpha, beta, kq, cn, rc, misc, raw gates
    static constexpr int RAW_OFF = ((SC_OFF + 8 * SC + 31) / 32) * 32;  // 128-byte aligned TMA boxes
    static constexpr int RAWK_B = SC * DK * 4, RAWV_B = SC * DV * 4;    // box bytes, fp32 worst case
    static constexpr int BAR_OFF = RAW_OFF + (2 * RAWK_B + RAWV_B) / 4;  // mbarrier (8 bytes)
    static constexpr size_t SMEM = sizeof(float) * (BAR_OFF + 4);
    static_assert(THREADS % 32 == 0, "whole warps (the tree shuffles use full masks)");
    static_assert(BAR_OFF % 2 == 0, "mbarrier alignment");
};

// The tensor maps of the q, k and v inputs ([T, H, D], box D x 1 x SC tokens).
struct TokMaps {
    const CUtensorMap* q;
    const CUtensorMap* k;
    const CUtensorMap* v;
};

// Barriers for a P_tok task: the whole CTA, or one 128-thread half of a
// larger CTA (named barrier `id`).
struct CtaSync {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};
struct HalfSync {
    int id;
    __device__ __forceinline__ void operator()() const { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }
};

// Set up a task context's mbarrier (thread 0 of the context; a barrier over
// the context must follow before the first task).
template <int DK, int DV, int C>
__device__ __forceinline__ void tok_context_init(float* sm, int tid)
{
    using Cf = TokCfg<DK, DV, C>;
    if (tid == 0) {
        mbar_init_cta(reinterpret_cast<uint64_t*>(sm + Cf::BAR_OFF), 1);
        sm[Cf::SC_OFF + 5 * Cf::SC + 2] = 0.0f;  // the abort flag: set once a wait runs out, never cleared
    }
}

// A 16-token sub-chunk with no fold: two blocks of 8 tokens, each fully
// unrolled with compile-time shared-memory offsets (no branch inside).
template <int DK, int DV, int RHO>
__device__ __forceinline__ void tok_sub16(f2x (&R)[RHO][DK / kLeaves], const float* kqb, const float* vsb,
                                          const float* scs, float* osb, bool write_o)
{
    using RS = RowSplit<DK>;
    constexpr int KS = RS::KS, SC = 16, HB = 8;
    f2x ax[RHO], ay[RHO], dd[RHO];
    tok_dots<DK, RHO>(R, kqb, kqb + KS, ax, ay);
#pragma unroll 1
    for (int hb = 0; hb < SC / HB; ++hb) {
        const float* kb = kqb + (hb * HB * 2) * KS;
        const float* vb = vsb + hb * HB * DV;
        const float* sb = scs + hb * HB;
        float* ob = osb + hb * HB * DV;
#pragma unroll
        for (int j = 0; j < HB; ++j) {
            float vv[RHO], oo[RHO];
            if constexpr (RHO == 4) {
                const float4 x = *reinterpret_cast<const float4*>(vb + j * DV);
                vv[0] = x.x; vv[1] = x.y; vv[2] = x.z; vv[3] = x.w;
            } else {
                const float2 x = *reinterpret_cast<const float2*>(vb + j * DV);
                vv[0] = x.x; vv[1] = x.y;
            }
            const float b = sb[SC + j], kq = sb[2 * SC + j], cn = sb[3 * SC + j], rc = sb[4 * SC + j];
#pragma unroll
            for (int r = 0; r < RHO; ++r) {
                float la, lb;
                up2(ax[r], la, lb);
                const float dk = tree_4lanes(la, lb);
                up2(ay[r], la, lb);
                const float dq = tree_4lanes(la, lb);
                const float dt = tok_scalars(dk, dq, vv[r], b, kq, cn, rc, false, oo[r]);
                dd[r] = pk2(dt, dt);
            }
            if (write_o) {
                if constexpr (RHO == 4) *reinterpret_cast<float4*>(ob + j * DV) = make_float4(oo[0], oo[1], oo[2], oo[3]);
                else *reinterpret_cast<float2*>(ob + j * DV) = make_float2(oo[0], oo[1]);
            }
            const float* kt = kb + (j * 2) * KS;
            if (j + 1 < HB || hb + 1 < SC / HB) tok_update_dots<DK, RHO>(R, dd, kt, kt + 2 * KS, kt + 3 * KS, ax, ay);
            else tok_update<DK, RHO>(R, dd, kt);
        }
    }
}

// Intra-chunk recurrence for chunk c of sequence n (tokens seq0 + cC ..), head
// h, by TokCfg::THREADS threads (tid = 0..THREADS-1) with smem `sm` of
// TokCfg::SMEM bytes (its mbarrier set up by tok_context_init; `phase` is the
// mbarrier's next phase parity, carried from task to task).  The chunk starts
// from states[slot] with scale 1 (COHERENT: read through L2, for states
// written earlier in the same launch).  For a partial last chunk the running
// state (Rt, c) goes to cacheR / cacheRs when non-null.  A TMA wait that runs
// out records GDN_ERR_TIMEOUT in *err and returns false.
template <int DK, int DV, int C, bool COHERENT, typename Sync>
__device__ __forceinline__ bool tok_task(const TokMaps maps, const float* __restrict__ alpha,
                                         const float* __restrict__ beta, int n, int c, int h, int H, int seq0, int Ln,
                                         int64_t slot, int in_bf16, int out_bf16, const float* states,
                                         void* __restrict__ o, float* __restrict__ cacheR, float* __restrict__ cacheRs,
                                         float* sm, int tid, Sync sync, uint32_t& phase, int32_t* err)
{
    using Cf = TokCfg<DK, DV, C>;
    using RS = typename Cf::RS;
    constexpr int RHO = Cf::RHO, SC = Cf::SC, L = RS::L, KS = RS::KS, NT = Cf::THREADS;
    float* kq = sm + Cf::KQ_OFF;
    float* vs = sm + Cf::VS_OFF;
    float* os = sm + Cf::OS_OFF;
    float* scs = sm + Cf::SC_OFF;
    float* al_s = scs;
    float* be_s = scs + SC;
    float* kq_s = scs + 2 * SC;
    float* cn_s = scs + 3 * SC;
    float* rc_s = scs + 4 * SC;
    float* misc = scs + 5 * SC;  // [0]: the scale carried between sub-chunks; [1]: fold mask; [2]: abort
    float* rab = scs + 6 * SC;   // [2][SC] gates as they arrive
    unsigned char* rawb = reinterpret_cast<unsigned char*>(sm + Cf::RAW_OFF);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Cf::BAR_OFF);

    const int64_t tok0 = (int64_t)seq0 + (int64_t)c * C;
    const int len = min(C, Ln - c * C);
    const int esz = in_bf16 ? 2 : 4;
    const int kbytes = DK * esz, vbytes = DV * esz;
    unsigned char* rawk = rawb;
    unsigned char* rawq = rawb + SC * kbytes;
    unsigned char* rawv = rawb + 2 * SC * kbytes;

    // sub-chunk s: k, q, v boxes by TMA (thread 0), the gates by cp.async
    auto fetch = [&](int s) {
        const int t0 = s * SC, ls = min(SC, len - t0);
        if (tid == 0) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(bar, (uint32_t)(SC * (2 * kbytes + vbytes)));
            tma_load_tokens(rawk, maps.k, h, (int)(tok0 + t0), bar);
            tma_load_tokens(rawq, maps.q, h, (int)(tok0 + t0), bar);
            tma_load_tokens(rawv, maps.v, h, (int)(tok0 + t0), bar);
        }
        for (int t = tid; t < ls; t += NT) {
            cp_async4(rab + t, alpha + (tok0 + t0 + t) * H + h);
            cp_async4(rab + SC + t, beta + (tok0 + t0 + t) * H + h);
        }
        cp_async_commit();
    };
    // raw sub-chunk -> fp32: k, q in the slot layout, v by row, gates.  Each
    // thread keeps one 8-element column group (NT is a multiple of the group
    // counts), so its slot offsets are computed once.
    constexpr int GK = DK / 8, GV = DV / 8;
    static_assert(NT % GK == 0 && NT % GV == 0, "fixed column groups per thread");
    int kslot[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) kslot[m] = RS::slot(8 * (tid % GK) + m);
    auto widen = [&](int ls) {
        const int gk = tid % GK, gv = tid % GV;
        for (int t = tid / GK; t < ls; t += NT / GK) {
            float x[8], y[8];
            lds8_raw(rawk + t * kbytes, 8 * gk, in_bf16, x);
            lds8_raw(rawq + t * kbytes, 8 * gk, in_bf16, y);
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                kq[(t * 2) * KS + kslot[m]] = x[m];
                kq[(t * 2 + 1) * KS + kslot[m]] = y[m];
            }
        }
        for (int t = tid / GV; t < ls; t += NT / GV) {
            float x[8];
            lds8_raw(rawv + t * vbytes, 8 * gv, in_bf16, x);
            *reinterpret_cast<float4*>(vs + t * DV + 8 * gv) = make_float4(x[0], x[1], x[2], x[3]);
            *reinterpret_cast<float4*>(vs + t * DV + 8 * gv + 4) = make_float4(x[4], x[5], x[6], x[7]);
        }
        for (int t = tid; t < ls; t += NT) {
            al_s[t] = rab[t];
            be_s[t] = rab[SC + t];
        }
    };

    const int gi = tid / RS::TPR, p = tid % RS::TPR;
    const int row0 = gi * RHO;
    f2x Rp[RHO][L];
#pragma unroll
    for (int r = 0; r < RHO; ++r) {
        const float* src = states + ((slot * H + h) * DV + row0 + r) * DK + p * RS::EPT;
        float t[RS::EPT];
#pragma unroll
        for (int e = 0; e < RS::EPT; e += 4) {
            const float4 x = COHERENT ? __ldcg(reinterpret_cast<const float4*>(src + e))
                                      : *reinterpret_cast<const float4*>(src + e);
            t[e] = x.x; t[e + 1] = x.y; t[e + 2] = x.z; t[e + 3] = x.w;
        }
#pragma unroll
        for (int m = 0; m < L; ++m) Rp[r][m] = pk2(t[m], t[L + m]);
    }
    if (tid == 0) misc[0] = 1.0f;

    const int nsub = (len + SC - 1) / SC;
    fetch(0);
    for (int s = 0; s < nsub; ++s) {
        const int ls = min(SC, len - s * SC);
        if (!mbar_wait_bounded(bar, phase, kWaitLimit)) misc[2] = 1.0f;
        phase ^= 1u;
        cp_async_wait_all();
        sync();  // raw(s) landed (or the wait ran out); the previous sub-chunk's outputs are stored
        if (misc[2] != 0.0f) {
            if (tid == 0) record_error(err, GDN_ERR_TIMEOUT);
            return false;
        }
        widen(ls);
        sync();  // fp32 buffers ready; raw is free again
        if (s + 1 < nsub) fetch(s + 1);
        // tree(k_t, q_t) of every token: 4 lanes per token
        for (int tt0 = 0; tt0 < SC; tt0 += NT / 4) {
            if (tid < 4 * SC) {
                const int tt = tt0 + (tid >> 2), pp = tid & 3;
                const float x = tok_kq<DK>(kq + (tt * 2) * KS + pp * RS::PS, kq + (tt * 2 + 1) * KS + pp * RS::PS);
                if (pp == 0 && tt < ls) kq_s[tt] = x;
            }
        }
        if (tid == 0) {  // the scale chain and this sub-chunk's folds (from the gates alone)
            float cs = misc[0];
            int mask = 0;
            for (int t = 0; t < ls; ++t) {
                const float cn = fmul(al_s[t], cs);
                const bool fold = !(cn >= kFoldTau);
                cn_s[t] = cn;
                mask |= fold ? (1 << t) : 0;
                cs = fold ? 1.0f : cn;
            }
            misc[0] = cs;
            misc[1] = __int_as_float(mask);
        }
        sync();
        if (tid < ls) rc_s[tid] = (__float_as_int(misc[1]) >> tid) & 1 ? 1.0f : __frcp_rn(cn_s[tid]);
        sync();
        const int mask = __float_as_int(misc[1]);
        const float* kqb = kq + p * RS::PS;
        if (mask == 0 && ls == SC) {
            tok_sub16<DK, DV, RHO>(Rp, kqb, vs + row0, scs, os + row0, p == 0);
        } else {
            f2x ax[RHO], ay[RHO], dd[RHO];
            tok_dots<DK, RHO>(Rp, kqb, kqb + KS, ax, ay);
            for (int t = 0; t < ls; ++t) {
                const bool fold = (mask >> t) & 1;
                const float cn = cn_s[t], rc = rc_s[t], bt = be_s[t], kqt = kq_s[t];
#pragma unroll
                for (int r = 0; r < RHO; ++r) {
                    float la, lb;
                    up2(ax[r], la, lb);
                    const float dk = tree_4lanes(la, lb);
                    up2(ay[r], la, lb);
                    const float dq = tree_4lanes(la, lb);
                    float ov;
                    const float dt = tok_scalars(dk, dq, vs[t * DV + row0 + r], bt, kqt, cn, rc, fold, ov);
                    dd[r] = pk2(dt, dt);
                    if (p == 0) os[t * DV + row0 + r] = ov;
                }
                if (fold) tok_scale<DK, RHO>(Rp, cn);
                const float* kt = kqb + (t * 2) * KS;
                if (t + 1 < ls) tok_update_dots<DK, RHO>(Rp, dd, kt, kt + 2 * KS, kt + 3 * KS, ax, ay);
                else tok_update<DK, RHO>(Rp, dd, kt);
            }
        }
        sync();
        for (int e = tid; e < ls * (DV / 8); e += NT) {
            const int t = e / (DV / 8), i8 = (e % (DV / 8)) * 8;
            store8(o, ((tok0 + s * SC + t) * H + h) * (int64_t)DV + i8, out_bf16, os + t * DV + i8);
        }
    }

    if (cacheR != nullptr && len < C) {  // last, partial chunk: the running state (Rt, c) for decode
#pragma unroll
        for (int r = 0; r < RHO; ++r)
            store_row_pairs<DK>(cacheR + (((int64_t)n * H + h) * DV + row0 + r) * DK + p * RS::EPT, Rp[r]);
        if (tid == 0) cacheRs[(int64_t)n * H + h] = misc[0];
    }
    sync();  // smem free for the next task
    return true;
}

// Intra-chunk recurrence: one CTA per (chunk task, head).
template <int DK, int DV, int C>
__global__ void __launch_bounds__(TokCfg<DK, DV, C>::THREADS)
k_tok(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
      const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ alpha, const float* __restrict__ beta,
      const int32_t* __restrict__ cu, const int32_t* __restrict__ cto, const int32_t* __restrict__ so, int32_t* err,
      int N, int H, int in_bf16, int out_bf16, const float* __restrict__ states, void* __restrict__ o,
      float* __restrict__ cacheR, float* __restrict__ cacheRs)
{
    if (*reinterpret_cast<volatile int32_t*>(err)) return;
    extern __shared__ __align__(128) float4 smem_a128[];  // TMA boxes need 128-byte alignment
    float* sm = reinterpret_cast<float*>(smem_a128);
    tok_context_init<DK, DV, C>(sm, threadIdx.x);
    __syncthreads();
    const int h = blockIdx.x % H;
    const int g = blockIdx.x / H;
    const int n = find_seq(cto, N, g);
    const int c = g - __ldg(cto + n);
    const int seq0 = __ldg(cu + n);
    uint32_t phase = 0;
    tok_task<DK, DV, C, false>(TokMaps{&tm_q, &tm_k, &tm_v}, alpha, beta, n, c, h, H, seq0,
                               __ldg(cu + n + 1) - seq0, (int64_t)__ldg(so + n) + c, in_bf16, out_bf16, states, o,
                               cacheR, cacheRs, sm, threadIdx.x, CtaSync{}, phase, err);
}

}  // namespace gdn
