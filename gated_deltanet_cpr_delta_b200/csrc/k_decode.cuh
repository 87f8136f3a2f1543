// k_decode.cuh -- decode step: k_dec_tok and k_dec_resync (sm_100a).
#pragma once

#include "k_ptok.cuh"
#include "k_pchunk.cuh"

namespace gdn {

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
    // the state rows are the bulk of the traffic: issue their loads before staging the token
    const int row = threadIdx.x / RS::TPR, part = threadIdx.x % RS::TPR;
    const int grow = r * Cf::RT + row;
    float* Rrow = R + ((int64_t)nh * DV + grow) * DK + part * RS::EPT;
    f2x Rp[RS::L];
    load_row_pairs<DK>(Rp, Rrow);
    stage_rows<DK>(ks, RS::KS, k, nh, 1, 1, 0, in_bf16, IdxSlot<DK>());
    stage_rows<DK>(qs, RS::KS, q, nh, 1, 1, 0, in_bf16, IdxSlot<DK>());
    for (int e = threadIdx.x; e < Cf::RT / 8; e += blockDim.x) {
        float x[8];
        load8(v, (int64_t)nh * DV + r * Cf::RT + e * 8, in_bf16, x);
#pragma unroll
        for (int m = 0; m < 8; ++m) vs[e * 8 + m] = x[m];
    }
    const float a = __ldg(alpha + nh), b = __ldg(beta + nh);
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
    using PL = PrepLayout<DK, DV, C>;
    using T = TcCfg<DK, DV, C>;
    static constexpr int KX_OFF = 0;                                 // [C][KXS] k, then w
    static constexpr int VX_OFF = KX_OFF + C * PL::KXS;              // [C][VXS] v, then u0
    static constexpr int WLO_OFF = VX_OFF + C * PL::VXS;             // canonical w lo, then w hi ...
    static constexpr int CC_OFF = WLO_OFF + T::W_FLOATS;             // ... in the [C][CCS] c of chunk_prep
    static constexpr int DM_OFF = CC_OFF + C * PL::CCS;              // decays / staging
    static constexpr int D0_OFF = DM_OFF + ((PL::DM + 3) / 4) * 4;   // D[t][0]
    static constexpr int AB_OFF = D0_OFF + C + 4;
    static constexpr int DC_OFF = AB_OFF + 2 * C;
    static constexpr int KLO_OFF = DC_OFF + Cf::DCS;                 // canonical k^T lo | hi, then S' staging
    static constexpr int KHI_OFF = KLO_OFF + T::K_FLOATS;
    static constexpr int BAR_OFF = KLO_OFF + T::K_REGION;            // mbarrier (8 bytes) + TMEM base
    // at least 120 KB, so that one CTA fits per SM: each allocates all 512 TMEM columns
    static constexpr size_t USED = sizeof(float) * (BAR_OFF + 4);
    static constexpr size_t BYTES = USED > 120 * 1024 ? USED : 120 * 1024;
    static_assert(BYTES <= 232448, "fits the 227 KB of shared memory a CTA can have");
    static_assert(D0_OFF - CC_OFF >= T::W_FLOATS, "w hi fits in the c / decay scratch");
    static_assert(BAR_OFF % 2 == 0 && DC_OFF % 4 == 0 && KLO_OFF % 4 == 0, "alignment");
};

// Advances pos after k_dec_tok appended a token at slot pos, and resyncs
// where that token completed a chunk: S_b <- P_chunk(S_b, buffer), R <- S_b,
// pos <- 0.  P_chunk runs the same device functions as the prefill
// (chunk_prep, then the tcgen05 boundary step).  Persistent: CTA b handles
// (sequence, head) pairs b, b + grid, ...  A pos outside [0, C) is left
// unchanged.  If an MMA completion wait times out, the pairs this CTA had
// still to resync get pos = -1 and are not written.
template <int DK, int DV, int C>
__global__ void __launch_bounds__(256, 1)
k_dec_resync(int NH, int in_bf16, float* S_b, float* R, const void* kbuf, const void* vbuf, const float* abuf,
             const float* bbuf, int32_t* pos)
{
    using Sm = ResyncSmem<DK, DV, C>;
    using PL = PrepLayout<DK, DV, C>;
    using T = TcCfg<DK, DV, C>;
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    float* kx = sm + Sm::KX_OFF;
    float* vx = sm + Sm::VX_OFF;
    float* cc = sm + Sm::CC_OFF;
    float* dm = sm + Sm::DM_OFF;
    float* d0 = sm + Sm::D0_OFF;
    float* as = sm + Sm::AB_OFF;
    float* bs = as + C;
    float* dCs = sm + Sm::DC_OFF;
    float* Wlo = sm + Sm::WLO_OFF;
    float* Whi = cc;  // == Wlo + C * DK
    float* Khi = sm + Sm::KHI_OFF;
    float* Klo = sm + Sm::KLO_OFF;
    uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + Sm::BAR_OFF);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Sm::BAR_OFF + 2);

    // this CTA's pairs are blockIdx.x + i*gridDim.x: read all their positions
    // at once, advance the ones inside a chunk, and list the ones at a boundary
    __shared__ int todo[1024];
    __shared__ int ntodo;
    if (threadIdx.x == 0) ntodo = 0;
    __syncthreads();
    for (int nh = blockIdx.x + threadIdx.x * gridDim.x; nh < NH; nh += blockDim.x * gridDim.x) {
        const int p = pos[nh];
        if (p < 0 || p >= C) continue;          // invalid: left unchanged
        if (p + 1 < C) {
            pos[nh] = p + 1;
        } else {
            const int slot = atomicAdd(&ntodo, 1);
            if (slot < 1024) todo[slot] = nh;   // the host sizes the grid so that a CTA has <= 1024 pairs
        }
    }
    __syncthreads();
    const int nt = min(ntodo, 1024);
    if (nt == 0) return;

    if (threadIdx.x == 0) mbar_init(mbar, 1);
    if (threadIdx.x < 32) tmem_alloc(tslot, T::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;
    const TcThread<DK> th(tbase);
    uint32_t parity = 0;
    float SR[DK / 2];
    int it = 0;
    for (; it < nt; ++it) {
        const int nh = todo[it];
        // buffer rows are [nh][slot][D]: a [T, H=1, D] tensor starting at token nh*C
        stage_rows<DK>(kx, PL::KXS, kbuf, (int64_t)nh * C, C, 1, 0, in_bf16, IdxIdentity());
        stage_rows<DV>(vx, PL::VXS, vbuf, (int64_t)nh * C, C, 1, 0, in_bf16, IdxIdentity());
        tc_stage_kT<DK, DV, C>(kbuf, (int64_t)nh * C, 1, 0, in_bf16, Khi, Klo);
        for (int t = threadIdx.x; t < C; t += blockDim.x) {
            as[t] = abuf[(int64_t)nh * C + t];
            bs[t] = bbuf[(int64_t)nh * C + t];
        }
        __syncthreads();
        chunk_prep<DK, DV, C>(kx, vx, as, bs, cc, dm, d0, in_bf16, kx, PL::KXS, vx, PL::VXS, dCs);
        tc_stage_w<DK, DV, C>(kx, PL::KXS, Whi, Wlo, threadIdx.x, blockDim.x);
        float* Sg = S_b + (int64_t)nh * DV * DK;
        tc_load_state<DK, DV, C>(SR, th, Sg, nullptr);
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (!tc_step<DK, DV, C>(SR, th, tbase, mbar, parity, Wlo, Klo, vx, PL::VXS, dCs, in_bf16, Sg,
                                R + (int64_t)nh * DV * DK))
            break;
        if (threadIdx.x == 0) pos[nh] = 0;
    }
    for (int r = it + threadIdx.x; r < nt; r += blockDim.x) pos[todo[r]] = -1;  // after a timeout
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(tbase, T::TMEM_COLS);
    }
}


}  // namespace gdn
