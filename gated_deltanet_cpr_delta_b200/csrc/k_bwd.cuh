// k_bwd.cuh -- CPR backward: gradients of L = sum_t dO_t . o_t (sm_100a).
//
// Reverse-mode differentiation of the token recurrence of the gated delta rule
// (IsoExec summary page, section "Chunkwise-Parallel Recurrent (CPR) Gated
// DeltaNet"; commentary blog, section 10).  With u = S_{t-1} k_t,
// delta = beta_t (v_t - alpha_t u), S_t = alpha_t S_{t-1} + delta k_t^T and
// G = dL/dS_t, one token backward is
//
//     G       += dO_t q_t^T
//     dq_t     = S_t^T dO_t                       ddelta = G k_t
//     dv_t     = beta_t ddelta                    dbeta_t = ddelta . (v_t - alpha_t u)
//     dalpha_t = <G, S_{t-1}> - beta_t ddelta . u
//     dk_t     = G^T delta - alpha_t beta_t S_{t-1}^T ddelta
//     G       <- alpha_t G - alpha_t beta_t ddelta k_t^T      (= dL/dS_{t-1})
//
// The backward keeps the forward's CPR split.  The G recursion does not need
// the forward states, so one light serial pass (k_bwd_scan) carries G from
// the last token to the first and stores it at every chunk boundary.  Then
// every chunk is independent: k_bwd_chunk starts from the boundary G after the
// chunk, recomputes the chunk's states from the forward's boundary state
// (one checkpoint per SUB tokens in a per-CTA global scratch, the current one
// and its midpoint in shared memory) and runs the per-token backward above.  Every row i of S and G evolves on its
// own, so both kernels split d_v into row tiles; dq, dk, dalpha and dbeta sum
// over rows, and the tiles' sums are added in a fixed order by k_bwd_reduce,
// so the gradients are deterministic.  Everything is fp32.
#pragma once

#include "k_ptok.cuh"

namespace gdn {

template <int DK, int DV, int C>
struct BwdCfg {
    using RS = RowSplit<DK>;
    static constexpr int RHO = 2;                 // rows per lane (k, q reads and row sums serve both)
    static constexpr int RT = DV < 64 ? DV : 64;  // rows per CTA
    static constexpr int NT = DV / RT;            // row tiles per head
    static constexpr int NG = RT / RHO;           // row groups (4 lanes each)
    static constexpr int THREADS = NG * RS::TPR;
    static constexpr int SUB = C < 8 ? C : 8;     // tokens per checkpoint
    static constexpr int NCK = C / SUB;           // checkpoints per chunk
    // staged floats per token: k, q (slots), v, dO rows, gates; a multiple of 4 (16-byte rows)
    static constexpr int TOKF = ((2 * RS::KS + 2 * RT + 2) + 3) / 4 * 4;
    static constexpr int RED = DK + 4;            // reduction buffer row stride
    // smem: SUB staged tokens | dq rows | dk rows | [NG][2] scalars | two lane-private state slots
    static constexpr int TOK_OFF = 0;
    static constexpr int RQ_OFF = TOK_OFF + SUB * TOKF;
    static constexpr int RK_OFF = RQ_OFF + NG * RED;
    static constexpr int RS_OFF = RK_OFF + NG * RED;
    static constexpr int CK_OFF = (RS_OFF + 2 * NG + 3) / 4 * 4;
    // two lane-private state slots (the sub-chunk's checkpoint and its
    // midpoint): a lane's RHO row slices, CKS floats, its 16-byte pieces
    // XOR-swizzled by the lane index so that 8 consecutive lanes reading the
    // same piece hit distinct banks
    static constexpr int CKS = RHO * RS::EPT;
    static constexpr int CK_PIECES = CKS / 4;
    static constexpr int CK_SWZ = (CK_PIECES < 8 ? CK_PIECES : 8) - 1;
    static constexpr int MID = SUB / 2;           // tokens from the checkpoint to the midpoint slot
    static constexpr size_t SMEM = sizeof(float) * (size_t)(CK_OFF + 2 * THREADS * CKS);
    static constexpr int64_t SCRATCH = (int64_t)NCK * RT * DK;  // floats of checkpoints per CTA
    static_assert(THREADS % 32 == 0, "whole warps (the tree shuffles use full masks)");
};

// Dot product of two lane shares of rows over all DK columns, every lane of
// the row getting the sum: up to 4 independent partial chains (the backward
// has no bitwise contract, so the order is free), then the 4-lane tree.
template <int DK>
__device__ __forceinline__ float row_dot(const f2x (&x)[DK / kLeaves], const f2x (&y)[DK / kLeaves])
{
    constexpr int L = DK / kLeaves;
    constexpr int NA = L < 4 ? L : 4;
    f2x acc[NA];
#pragma unroll
    for (int j = 0; j < NA; ++j) acc[j] = fmul2(x[j], y[j]);
#pragma unroll
    for (int m = NA; m < L; ++m) acc[m % NA] = ffma2(x[m], y[m], acc[m % NA]);
    float la = 0.f, lb = 0.f;
#pragma unroll
    for (int j = 0; j < NA; ++j) {
        float a, b;
        up2(acc[j], a, b);
        la = j == 0 ? a : fadd(la, a);
        lb = j == 0 ? b : fadd(lb, b);
    }
    return tree_4lanes(la, lb);
}

template <int DK>
__device__ __forceinline__ void load_pairs_slot(f2x (&p)[DK / kLeaves], const float* s)
{
    constexpr int L = DK / kLeaves;
#pragma unroll
    for (int m = 0; m < L; m += 2) {
        const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(s + 2 * m);
        p[m] = x.x;
        p[m + 1] = x.y;
    }
}

// Serial pass over one (sequence, head, row tile): G from the last token
// (starting from the final state's gradient, or zero) to the first, without
// the gradient outputs.  After the chunk starting at token c*C it holds
// Y_c = dL/dS(c*C) through the tokens >= c*C; Y_c (c >= 1) goes to ybuf at
// the chunk-state slot so[n] + c, Y_0 = dL/dstate_in to dstate.
// Tokens are staged raw (bf16 or fp32) by cp.async in blocks of BLK, NBUF
// blocks in flight; each lane widens its own slice.  The lane's EPT columns
// are held as pairs of adjacent columns.  (Widening a bf16 block once into an
// fp32 buffer measured slower: the extra pass and barrier sit on the serial
// path.)
template <int DK, int DV, int C>
struct ScanCfg {
    static constexpr int RT = DV < 32 ? DV : 32;
    static constexpr int NT = DV / RT;
    static constexpr int TPR = 4;
    static constexpr int EPT = DK / TPR;
    static constexpr int NP = EPT / 2;
    static constexpr int THREADS = RT * TPR;
    static constexpr int BLK = 16;
    static constexpr int NBUF = 3;
    static_assert(C % BLK == 0, "chunks are whole blocks");
    template <int ES>
    struct L {
        static constexpr int PAD = EPT * ES >= 16 ? 16 : 0;   // keeps the 4 lanes' slices in distinct banks
        static constexpr int PSB = EPT * ES + PAD;            // bytes between the lanes' slices
        static constexpr int ROWB = TPR * PSB;                // one q or k row
        static constexpr int DOB = RT * ES;                   // this tile's dO row
        static constexpr int GOFF = 2 * ROWB + DOB;           // alpha, beta
        static constexpr int TOKB = (GOFF + 8 + 15) / 16 * 16;
        static constexpr int STAGE = BLK * TOKB;
    };
    static constexpr size_t SMEM = (size_t)NBUF * L<4>::STAGE;
};

template <int ES, int NP>
__device__ __forceinline__ void widen_pairs(f2x (&p)[NP], const unsigned char* s)
{
    if constexpr (ES == 2) {
        static_assert(NP % 2 == 0, "");
#pragma unroll
        for (int m = 0; m < NP; m += 2) {
            const uint2 w = *reinterpret_cast<const uint2*>(s + 2 * 2 * m);
            p[m] = pk2(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u));
            p[m + 1] = pk2(__uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
        }
    } else {
#pragma unroll
        for (int m = 0; m < NP; m += 2) {
            const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(s + 4 * 2 * m);
            p[m] = x.x;
            p[m + 1] = x.y;
        }
    }
}

template <int DK, int DV, int C, int ES>
__device__ __forceinline__ void bwd_scan_body(const void* q, const void* k, const float* alpha, const float* beta,
                                              const void* dO, int seq0, int Ln, int64_t slot0, int h, int H, int r,
                                              const float* gfinal_row, float* ybuf, float* dstate_row,
                                              unsigned char* sm)
{
    using Cf = ScanCfg<DK, DV, C>;
    using Lt = typename Cf::template L<ES>;
    constexpr int NP = Cf::NP, EPT = Cf::EPT, RT = Cf::RT, BLK = Cf::BLK, NBUF = Cf::NBUF;
    constexpr int QCH = DK * ES / 16;  // 16-byte pieces of a q / k row
    constexpr int DCH = RT * ES / 16;  // of this tile's dO row
    const int tid = threadIdx.x;
    const int row = tid / Cf::TPR, part = tid % Cf::TPR;
    const int grow = r * RT + row;
    const char* qb = static_cast<const char*>(q);
    const char* kb = static_cast<const char*>(k);
    const char* db = static_cast<const char*>(dO);
    const int nblk = (Ln + BLK - 1) / BLK;

    auto issue = [&](int i) {
        if (i < nblk) {
            unsigned char* st = sm + (i % NBUF) * Lt::STAGE;
            const int t0 = (nblk - 1 - i) * BLK, len = min(BLK, Ln - t0);
            for (int e = tid; e < len * (2 * QCH + DCH + 2); e += blockDim.x) {
                const int t = e / (2 * QCH + DCH + 2), w = e % (2 * QCH + DCH + 2);
                const int64_t trow = ((int64_t)seq0 + t0 + t) * H + h;
                unsigned char* d = st + t * Lt::TOKB;
                if (w < 2 * QCH) {
                    const int j = w % QCH;
                    const int byte = j * 16;
                    const int dst = Lt::PAD ? (byte / (EPT * ES)) * Lt::PSB + byte % (EPT * ES) : byte;
                    cp_async16(d + (w < QCH ? 0 : Lt::ROWB) + dst, (w < QCH ? qb : kb) + trow * DK * ES + byte);
                } else if (w < 2 * QCH + DCH) {
                    const int j = w - 2 * QCH;
                    cp_async16(d + 2 * Lt::ROWB + j * 16, db + (trow * DV + r * RT) * ES + j * 16);
                } else {
                    cp_async4(d + Lt::GOFF + 4 * (w - 2 * QCH - DCH), (w == 2 * QCH + DCH ? alpha : beta) + trow);
                }
            }
        }
        cp_async_commit();
    };

    // G starts from the final state's gradient (zero without one)
    f2x G[NP];
    if (gfinal_row != nullptr) {
#pragma unroll
        for (int m = 0; m < NP; m += 2) {
            const float4 x = *reinterpret_cast<const float4*>(gfinal_row + part * EPT + 2 * m);
            G[m] = pk2(x.x, x.y);
            G[m + 1] = pk2(x.z, x.w);
        }
    } else {
#pragma unroll
        for (int m = 0; m < NP; ++m) G[m] = pk2(0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < NBUF - 1; ++i) issue(i);
    for (int i = 0; i < nblk; ++i) {
        cp_async_wait_n<NBUF - 2>();
        __syncthreads();
        issue(i + NBUF - 1);
        const unsigned char* st = sm + (i % NBUF) * Lt::STAGE;
        const int t0 = (nblk - 1 - i) * BLK, len = min(BLK, Ln - t0);
        for (int t = len - 1; t >= 0; --t) {
            const unsigned char* tk = st + t * Lt::TOKB;
            f2x qp[NP], kp[NP];
            widen_pairs<ES, NP>(qp, tk + part * Lt::PSB);
            widen_pairs<ES, NP>(kp, tk + Lt::ROWB + part * Lt::PSB);
            float doi;
            if constexpr (ES == 2)
                doi = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(tk + 2 * Lt::ROWB)[row] << 16);
            else
                doi = reinterpret_cast<const float*>(tk + 2 * Lt::ROWB)[row];
            const float a = *reinterpret_cast<const float*>(tk + Lt::GOFF);
            const float b = *reinterpret_cast<const float*>(tk + Lt::GOFF + 4);
            const f2x oo = pk2(doi, doi);
#pragma unroll
            for (int m = 0; m < NP; ++m) G[m] = ffma2(oo, qp[m], G[m]);
            f2x acc0 = fmul2(G[0], kp[0]), acc1 = fmul2(G[1], kp[1]);
#pragma unroll
            for (int m = 2; m < NP; m += 2) {
                acc0 = ffma2(G[m], kp[m], acc0);
                acc1 = ffma2(G[m + 1], kp[m + 1], acc1);
            }
            float l0, l1, l2, l3;
            up2(acc0, l0, l1);
            up2(acc1, l2, l3);
            const float dlt = tree_4lanes(fadd(l0, l2), fadd(l1, l3));
            const float ng = -fmul(fmul(a, b), dlt);
            const f2x aa = pk2(a, a), nn = pk2(ng, ng);
#pragma unroll
            for (int m = 0; m < NP; ++m) G[m] = ffma2(nn, kp[m], fmul2(aa, G[m]));
            const int tg = t0 + t;
            if (tg % C == 0) {
                float* dst = tg == 0 ? dstate_row : ybuf + (((slot0 + tg / C) * H + h) * DV + grow) * (int64_t)DK;
#pragma unroll
                for (int m = 0; m < NP; m += 2) {
                    float x0, x1, x2, x3;
                    up2(G[m], x0, x1);
                    up2(G[m + 1], x2, x3);
                    *reinterpret_cast<float4*>(dst + part * EPT + 2 * m) = make_float4(x0, x1, x2, x3);
                }
            }
        }
    }
    cp_async_wait_all();
    if (Ln == 0) {  // no tokens: dL/dstate_in is the final state's gradient
#pragma unroll
        for (int m = 0; m < NP; m += 2) {
            float x0, x1, x2, x3;
            up2(G[m], x0, x1);
            up2(G[m + 1], x2, x3);
            *reinterpret_cast<float4*>(dstate_row + part * EPT + 2 * m) = make_float4(x0, x1, x2, x3);
        }
    }
}

template <int DK, int DV, int C>
__global__ void __launch_bounds__(ScanCfg<DK, DV, C>::THREADS)
k_bwd_scan(const void* __restrict__ q, const void* __restrict__ k, const float* __restrict__ alpha,
           const float* __restrict__ beta, const void* __restrict__ dO, const int32_t* __restrict__ cu,
           const int32_t* __restrict__ so, const int32_t* __restrict__ err, int H, int in_bf16,
           const float* __restrict__ dstate_out, float* __restrict__ ybuf, float* __restrict__ dstate)
{
    using Cf = ScanCfg<DK, DV, C>;
    if (__ldg(err)) return;
    extern __shared__ float4 smem_f4[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(smem_f4);
    const int r = blockIdx.x % Cf::NT;
    const int nh = blockIdx.x / Cf::NT;
    const int h = nh % H, n = nh / H;
    const int seq0 = __ldg(cu + n);
    const int Ln = __ldg(cu + n + 1) - seq0;
    const int64_t slot0 = __ldg(so + n);
    const int row = threadIdx.x / Cf::TPR;
    const int64_t roff = ((int64_t)nh * DV + r * Cf::RT + row) * DK;
    float* dstate_row = dstate + roff;
    const float* gfinal_row = dstate_out != nullptr ? dstate_out + roff : nullptr;
    if (in_bf16)
        bwd_scan_body<DK, DV, C, 2>(q, k, alpha, beta, dO, seq0, Ln, slot0, h, H, r, gfinal_row, ybuf, dstate_row,
                                    sm);
    else
        bwd_scan_body<DK, DV, C, 4>(q, k, alpha, beta, dO, seq0, Ln, slot0, h, H, r, gfinal_row, ybuf, dstate_row,
                                    sm);
}

// One forward P_tok step (the forward's operations) on RHO rows of this lane
// that share the staged k_t.
template <int DK, int RHO>
__device__ __forceinline__ void adv_rows(f2x (&Sp)[RHO][DK / kLeaves], const float* kt, const float* vrow, float a,
                                         float b)
{
    constexpr int L = DK / kLeaves;
    f2x kp[L];
    load_pairs_slot<DK>(kp, kt);
    const f2x aa = pk2(a, a);
#pragma unroll
    for (int r = 0; r < RHO; ++r) {
        const float u = row_dot<DK>(Sp[r], kp);
        const float d = fmul(b, fsub(vrow[r], fmul(a, u)));
        const f2x dd = pk2(d, d);
#pragma unroll
        for (int m = 0; m < L; ++m) Sp[r][m] = ffma2(dd, kp[m], fmul2(aa, Sp[r][m]));
    }
}

// Stores 2*G4 floats of a lane's natural-order slice: elements m0..m0+G4-1
// from lo[], L+m0.. from hi[].
template <int G4>
__device__ __forceinline__ void st_group(float* dst, int m0, int L, const float* lo, const float* hi)
{
    if constexpr (G4 == 4) {
        *reinterpret_cast<float4*>(dst + m0) = make_float4(lo[0], lo[1], lo[2], lo[3]);
        *reinterpret_cast<float4*>(dst + L + m0) = make_float4(hi[0], hi[1], hi[2], hi[3]);
    } else {
        *reinterpret_cast<float2*>(dst + m0) = make_float2(lo[0], lo[1]);
        *reinterpret_cast<float2*>(dst + L + m0) = make_float2(hi[0], hi[1]);
    }
}

// A lane's RHO rows (natural column order) to / from its swizzled slot.
template <int DK, int RHO, int SWZ>
__device__ __forceinline__ void slot_store(float* slot, int sw, const f2x (&Sp)[RHO][DK / kLeaves])
{
    constexpr int L = DK / kLeaves, EPT = 2 * L;
#pragma unroll
    for (int r = 0; r < RHO; ++r) {
        float t[EPT];
#pragma unroll
        for (int m = 0; m < L; ++m) up2(Sp[r][m], t[m], t[L + m]);
#pragma unroll
        for (int e = 0; e < EPT; e += 4)
            *reinterpret_cast<float4*>(slot + 4 * (((r * EPT + e) >> 2) ^ (sw & SWZ))) =
                make_float4(t[e], t[e + 1], t[e + 2], t[e + 3]);
    }
}

template <int DK, int RHO, int SWZ>
__device__ __forceinline__ void slot_load(f2x (&Sp)[RHO][DK / kLeaves], const float* slot, int sw)
{
    constexpr int L = DK / kLeaves, EPT = 2 * L;
#pragma unroll
    for (int r = 0; r < RHO; ++r) {
        float t[EPT];
#pragma unroll
        for (int e = 0; e < EPT; e += 4) {
            const float4 x = *reinterpret_cast<const float4*>(slot + 4 * (((r * EPT + e) >> 2) ^ (sw & SWZ)));
            t[e] = x.x; t[e + 1] = x.y; t[e + 2] = x.z; t[e + 3] = x.w;
        }
#pragma unroll
        for (int m = 0; m < L; ++m) Sp[r][m] = pk2(t[m], t[L + m]);
    }
}

// Backward of the chunks: one (chunk, head, row tile) task at a time, CTAs
// looping over the tasks (a persistent grid, so that the checkpoint scratch
// is per resident CTA and stays in L2).  Each lane holds RHO rows (a quarter
// of each row's columns), so one read of a staged k or q serves RHO rows and
// the lane adds its rows' dq / dk terms before they go to shared memory.  A
// task starts from G = Y_{c+1} (zero after the last chunk), recomputes the
// chunk's states from its boundary state and writes dv rows, and the tile's
// row sums of dq, dk ([NT][T][H][DK]) and dalpha, dbeta ([NT][T][H]).  The
// last chunk of a sequence starts from the final state's gradient when given.
template <int DK, int DV, int C>
__global__ void __launch_bounds__(BwdCfg<DK, DV, C>::THREADS)
k_bwd_chunk(const void* __restrict__ q, const void* __restrict__ k, const void* __restrict__ v,
            const float* __restrict__ alpha, const float* __restrict__ beta, const void* __restrict__ dO,
            const float* __restrict__ states, const float* __restrict__ ybuf,
            const float* __restrict__ dstate_out, const int32_t* __restrict__ cu,
            const int32_t* __restrict__ cto, const int32_t* __restrict__ so, const int32_t* __restrict__ err,
            int N, int H, int64_t T_total, int64_t ntasks, int in_bf16, float* __restrict__ dv,
            float* __restrict__ pq, float* __restrict__ pk, float* __restrict__ pa, float* __restrict__ pb,
            float* __restrict__ scratch)
{
    using Cf = BwdCfg<DK, DV, C>;
    using RS = typename Cf::RS;
    constexpr int L = RS::L, KS = RS::KS, RT = Cf::RT, SUB = Cf::SUB, TOKF = Cf::TOKF, NT = Cf::NT;
    constexpr int RHO = Cf::RHO, NG = Cf::NG, EPT = RS::EPT;
    constexpr int G4 = L % 4 == 0 ? 4 : 2;
    static_assert(L % G4 == 0, "");
    if (__ldg(err)) return;
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    float* tok = sm + Cf::TOK_OFF;
    float* redq = sm + Cf::RQ_OFF;
    float* redk = sm + Cf::RK_OFF;
    float* reds = sm + Cf::RS_OFF;
    const int tid = threadIdx.x;
    const int gi = tid / RS::TPR, part = tid % RS::TPR;
    const int lrow0 = gi * RHO;  // this lane's first row in the tile
    float* slotA = sm + Cf::CK_OFF + tid * Cf::CKS;                 // the sub-chunk's checkpoint
    float* slotB = sm + Cf::CK_OFF + (Cf::THREADS + tid) * Cf::CKS;  // the state MID tokens later
    float* ck = scratch + (int64_t)blockIdx.x * Cf::SCRATCH;   // this CTA's checkpoints

    for (int64_t task = blockIdx.x; task < ntasks; task += gridDim.x) {
        const int rt = (int)(task % NT);
        const int h = (int)((task / NT) % H);
        const int ct = (int)(task / ((int64_t)NT * H));
        const int n = find_seq(cto, N, ct);
        const int c = ct - __ldg(cto + n);
        const int seq0 = __ldg(cu + n);
        const int Ln = __ldg(cu + n + 1) - seq0;
        const int64_t slot0 = __ldg(so + n);
        const int nchunks = (Ln + C - 1) / C;
        const int grow0 = rt * RT + lrow0;  // this lane's first row in the head

        // stage tokens [t0, t0 + len) of the sequence: k, q into the slot layout,
        // this tile's v and dO rows, the gates
        auto stage = [&](int t0, int len) {
            constexpr int G8 = (2 * DK) / 8;
            for (int e = tid; e < len * G8; e += blockDim.x) {
                const int t = e / G8, el = (e % G8) * 8;
                float x[8];
                const int64_t trow = ((int64_t)seq0 + t0 + t) * H + h;
                load8(el < DK ? k : q, trow * DK + (el % DK), in_bf16, x);
                float* d = tok + t * TOKF + (el >= DK ? KS : 0);
#pragma unroll
                for (int m = 0; m < 8; ++m) d[RS::slot((el % DK) + m)] = x[m];
            }
            for (int e = tid; e < len * (2 * RT / 8); e += blockDim.x) {
                const int t = e / (2 * RT / 8), el = (e % (2 * RT / 8)) * 8;
                float x[8];
                const int64_t trow = ((int64_t)seq0 + t0 + t) * H + h;
                load8(el < RT ? v : dO, trow * DV + rt * RT + (el % RT), in_bf16, x);
                float* d = tok + t * TOKF + 2 * KS + (el >= RT ? RT : 0) + (el % RT);
#pragma unroll
                for (int m = 0; m < 8; ++m) d[m] = x[m];
            }
            for (int t = tid; t < len; t += blockDim.x) {
                const int64_t trow = ((int64_t)seq0 + t0 + t) * H + h;
                tok[t * TOKF + 2 * KS + 2 * RT] = __ldg(alpha + trow);
                tok[t * TOKF + 2 * KS + 2 * RT + 1] = __ldg(beta + trow);
            }
        };
        auto step = [&](f2x (&Sp)[RHO][L], int t) {  // forward step with staged token t
            const float* tt = tok + t * TOKF;
            adv_rows<DK, RHO>(Sp, tt + part * RS::PS, tt + 2 * KS + lrow0, tt[2 * KS + 2 * RT],
                              tt[2 * KS + 2 * RT + 1]);
        };

        f2x G[RHO][L];
#pragma unroll
        for (int r = 0; r < RHO; ++r) {
            if (c + 1 < nchunks) {
                load_row_pairs<DK>(G[r], ybuf + (((slot0 + c + 1) * H + h) * DV + grow0 + r) * DK + part * EPT);
            } else if (dstate_out != nullptr) {  // the last chunk starts from the final state's gradient
                load_row_pairs<DK>(G[r], dstate_out + (((int64_t)n * H + h) * DV + grow0 + r) * DK + part * EPT);
            } else {
#pragma unroll
                for (int m = 0; m < L; ++m) G[r][m] = pk2(0.f, 0.f);
            }
        }
        const float* S0 = states + (((slot0 + c) * H + h) * DV + grow0) * DK + part * EPT;
        const int cb = c * C, clen = min(C, Ln - cb);
        const int nsub = (clen + SUB - 1) / SUB;
        // checkpoints: the state at cb + j*SUB, j = 1..nsub-1 (j = 0 is the chunk state)
        f2x Sp[RHO][L];
#pragma unroll
        for (int r = 0; r < RHO; ++r) load_row_pairs<DK>(Sp[r], S0 + r * DK);
        for (int j = 1; j < nsub; ++j) {
            __syncthreads();
            stage(cb + (j - 1) * SUB, SUB);
            __syncthreads();
            for (int t = 0; t < SUB; ++t) step(Sp, t);
#pragma unroll
            for (int r = 0; r < RHO; ++r)
                store_row_pairs<DK>(ck + ((int64_t)(j - 1) * RT + lrow0 + r) * DK + part * EPT, Sp[r]);
        }
        // backward over the sub-chunks, last first
        for (int j = nsub - 1; j >= 0; --j) {
            const int sb = cb + j * SUB, slen = min(SUB, clen - j * SUB);
            __syncthreads();
            stage(sb, slen);
            // the sub-chunk's checkpoint into this lane's slot A, and the state
            // MID tokens later into slot B (read back once per token)
#pragma unroll
            for (int r = 0; r < RHO; ++r) {
                const float* src = j == 0 ? S0 + r * DK : ck + ((int64_t)(j - 1) * RT + lrow0 + r) * DK + part * EPT;
                load_row_pairs<DK>(Sp[r], src);
            }
            slot_store<DK, RHO, Cf::CK_SWZ>(slotA, tid, Sp);
            __syncthreads();
            if (slen > Cf::MID) {
                for (int m = 0; m < Cf::MID; ++m) step(Sp, m);
                slot_store<DK, RHO, Cf::CK_SWZ>(slotB, tid, Sp);
            }
            for (int t = slen - 1; t >= 0; --t) {
                // S_{t-1}: from the nearer of the two slots, forward over the tokens in between
                const bool fromB = t >= Cf::MID;
                slot_load<DK, RHO, Cf::CK_SWZ>(Sp, fromB ? slotB : slotA, tid);
                for (int m = fromB ? Cf::MID : 0; m < t; ++m) step(Sp, m);
                const float* tt = tok + t * TOKF;
                const float a = tt[2 * KS + 2 * RT], b = tt[2 * KS + 2 * RT + 1];
                const f2x aa = pk2(a, a);
                const float ab = fmul(a, b);
                f2x kp[L];
                load_pairs_slot<DK>(kp, tt + part * RS::PS);
                float u[RHO], de[RHO], dlt[RHO], vi[RHO], doi[RHO];
                {
                    f2x qp[L];
                    load_pairs_slot<DK>(qp, tt + KS + part * RS::PS);
#pragma unroll
                    for (int r = 0; r < RHO; ++r) {
                        vi[r] = tt[2 * KS + lrow0 + r];
                        doi[r] = tt[2 * KS + RT + lrow0 + r];
                        const f2x oo = pk2(doi[r], doi[r]);
#pragma unroll
                        for (int m = 0; m < L; ++m) G[r][m] = ffma2(oo, qp[m], G[r][m]);  // G += dO_i q
                    }
                }
                float ta = 0.f, tb = 0.f;  // this lane's rows' dalpha and dbeta terms
#pragma unroll
                for (int r = 0; r < RHO; ++r) {
                    u[r] = row_dot<DK>(Sp[r], kp);
                    de[r] = fmul(b, fsub(vi[r], fmul(a, u[r])));
                    dlt[r] = row_dot<DK>(G[r], kp);        // ddelta_i
                    const float gs = row_dot<DK>(G[r], Sp[r]);  // <G_i, S_{t-1,i}>
                    ta = fadd(ta, fsub(gs, fmul(b, fmul(dlt[r], u[r]))));
                    tb = fadd(tb, fmul(dlt[r], fsub(vi[r], fmul(a, u[r]))));
                }
                // the lane's rows' dq terms (dO_i S_t) and dk terms (G delta - ab ddelta S_{t-1}),
                // added over its rows, to the reduction buffers in natural column order
#pragma unroll
                for (int m0 = 0; m0 < L; m0 += G4) {
                    float ql[G4], qh[G4], kl[G4], kh[G4];
#pragma unroll
                    for (int mm = 0; mm < G4; ++mm) {
                        const int m = m0 + mm;
                        f2x sq = pk2(0.f, 0.f), sk = pk2(0.f, 0.f);
#pragma unroll
                        for (int r = 0; r < RHO; ++r) {
                            const f2x dd = pk2(de[r], de[r]);
                            const f2x st = ffma2(dd, kp[m], fmul2(aa, Sp[r][m]));   // S_t
                            sq = ffma2(pk2(doi[r], doi[r]), st, sq);
                            const float nb = -fmul(ab, dlt[r]);
                            sk = ffma2(pk2(nb, nb), Sp[r][m], ffma2(dd, G[r][m], sk));
                        }
                        up2(sq, ql[mm], qh[mm]);
                        up2(sk, kl[mm], kh[mm]);
                    }
                    st_group<G4>(redq + gi * Cf::RED + part * EPT, m0, L, ql, qh);
                    st_group<G4>(redk + gi * Cf::RED + part * EPT, m0, L, kl, kh);
                }
                if (part == 0) {
                    reds[2 * gi] = ta;
                    reds[2 * gi + 1] = tb;
#pragma unroll
                    for (int r = 0; r < RHO; ++r)
                        dv[(((int64_t)seq0 + sb + t) * H + h) * DV + grow0 + r] = fmul(b, dlt[r]);
                }
                // G <- alpha G - alpha beta ddelta k
#pragma unroll
                for (int r = 0; r < RHO; ++r) {
                    const float nb = -fmul(ab, dlt[r]);
                    const f2x ng = pk2(nb, nb);
#pragma unroll
                    for (int m = 0; m < L; ++m) G[r][m] = ffma2(ng, kp[m], fmul2(aa, G[r][m]));
                }
                __syncthreads();
                // the tile's row-group sums, groups in ascending order
                const int64_t trow = ((int64_t)seq0 + sb + t) * H + h;
                for (int col = tid; col < 2 * DK; col += blockDim.x) {
                    const float* src = col < DK ? redq + col : redk + (col - DK);
                    float s = src[0];
                    for (int i = 1; i < NG; ++i) s = fadd(s, src[i * Cf::RED]);
                    float* dst = col < DK ? pq : pk;
                    dst[((int64_t)rt * T_total * H + trow) * DK + (col % DK)] = s;
                }
                if (tid < 2) {
                    float s = reds[tid];
                    for (int i = 1; i < NG; ++i) s = fadd(s, reds[2 * i + tid]);
                    (tid == 0 ? pa : pb)[(int64_t)rt * T_total * H + trow] = s;
                }
                __syncthreads();
            }
        }
    }
}

// dq, dk, dalpha, dbeta = the sum of the NT tiles' partials, tile 0 first.
template <int DK, int NT>
__global__ void k_bwd_reduce(const float* __restrict__ pq, const float* __restrict__ pk, const float* __restrict__ pa,
                             const float* __restrict__ pb, const int32_t* __restrict__ err, int64_t TH,
                             float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ da,
                             float* __restrict__ db)
{
    if (__ldg(err)) return;
    const int64_t nvec = TH * DK;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nvec + TH; i += (int64_t)gridDim.x * blockDim.x) {
        if (i < nvec) {
            float sq = pq[i], sk = pk[i];
#pragma unroll
            for (int r = 1; r < NT; ++r) {
                sq = fadd(sq, pq[r * nvec + i]);
                sk = fadd(sk, pk[r * nvec + i]);
            }
            dq[i] = sq;
            dk[i] = sk;
        } else {
            const int64_t j = i - nvec;
            float sa = pa[j], sb = pb[j];
#pragma unroll
            for (int r = 1; r < NT; ++r) {
                sa = fadd(sa, pa[r * TH + j]);
                sb = fadd(sb, pb[r * TH + j]);
            }
            da[j] = sa;
            db[j] = sb;
        }
    }
}

}  // namespace gdn
