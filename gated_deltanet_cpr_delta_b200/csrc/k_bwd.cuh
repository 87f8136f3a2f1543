// k_bwd.cuh -- CPR backward, the boundary adjoints (sm_100a).
//
// Reverse-mode differentiation of the token recurrence of the gated delta rule
// (IsoExec summary page, section "Chunkwise-Parallel Recurrent (CPR) Gated
// DeltaNet"; commentary blog, section 10).  With u = S_{t-1} k_t,
// delta = beta_t (v_t - alpha_t u), S_t = alpha_t S_{t-1} + delta k_t^T and
// G = dL/dS_t, the adjoint of the state runs backwards as
//
//     G <- alpha_t (G + dO_t q_t^T) - alpha_t beta_t ((G + dO_t q_t^T) k_t) k_t^T
//
// which needs no forward state.  k_bwd_scan carries G from each sequence's
// last token to its first and stores it at every chunk boundary; the
// per-chunk gradients (k_bprep, k_bgrad) start from those boundary adjoints.
#pragma once

#include "k_ptok.cuh"

namespace gdn {

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

}  // namespace gdn
