// k_pchunk.cuh -- chunk-boundary update P_chunk: k_prep, k_chain, k_cache_fill (sm_100a).
#pragma once

#include "k_ptok.cuh"
#include "k_tc.cuh"

namespace gdn {

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

// P_chunk part 1 for one chunk, by one CTA (>= 128 threads), on the tensor
// cores where the work is a dense contraction:
//   D[s][s] = 1, D[t][s] = D[t-1][s] * alpha_t                     (fp32 chains)
//   G[t][s] = k_t . k_s for s < t: mma tf32 over 8-wide blocks of d_k,
//             ascending, k = k_hi + k_lo (k_lo = 0 and skipped when every k
//             is exactly tf32, i.e. bf16 inputs):  G += k_lo*k_hi, k_hi*k_lo, k_hi*k_hi
//   c[t][s] = D[t][s] * G[t][s]
//   forward substitution for the columns x = u0 (init v_t) and w (init
//   D[t][0] * k_t), in blocks of 16 tokens: for block b, acc_t = init_t;
//   acc_t += sum over 8-token blocks of s < 16b (ascending) of the mma
//   products (-c)_lo*x_hi, (-c)_hi*x_lo, (-c)_hi*x_hi; then, for s in
//   [16b, t) ascending, acc_t = fma(-c[t][s], x_s, acc_t); x_t = beta_t * acc_t.
// kx [C][DK+8] holds k on entry and w on exit; vx [C][DV+8] holds v on entry
// and u0 on exit (row strides chosen so the mma fragment reads are
// conflict-free); as, bs [C] gates; cc [C][C+4], dm, d0 are smem scratch.
// Also writes w -> wout[t*ldw + j], u0 -> uout[t*ldu + i], D[C][s] -> dCout[s]
// (any address space; uout may be vx itself).
template <int DK, int DV, int C>
struct PrepLayout {
    static constexpr int KXS = DK + 8, VXS = DV + 8, CCS = C + 4;
    static constexpr int NCOL = DV + DK;
    static constexpr int STS = NCOL + 8;  // staging row stride: conflict-free fragment stores
    static constexpr int DM = ((C + 1) * (C + 1) > 16 * STS ? (C + 1) * (C + 1) : 16 * STS);
};

template <int DK, int DV, int C>
__device__ __forceinline__ void chunk_prep(float* kx, float* vx, const float* as, const float* bs, float* cc, float* dm,
                                           float* d0, int k_exact, float* wout, int ldw, float* uout, int ldu,
                                           float* dCout)
{
    using PL = PrepLayout<DK, DV, C>;
    constexpr int KXS = PL::KXS, VXS = PL::VXS, CCS = PL::CCS, C1 = C + 1, NCOL = PL::NCOL, STS = PL::STS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
    const int nwarps = blockDim.x >> 5;
    // decay products: column s is the chain D[t][s] = D[t-1][s] * alpha_t, t = s+1..C
    for (int s = threadIdx.x; s <= C; s += blockDim.x) {
        float d = 1.0f;
        dm[s * C1 + s] = d;
#pragma unroll
        for (int t4i = 0; t4i < C; t4i += 4) {
            const float4 a4 = *reinterpret_cast<const float4*>(as + t4i);
            const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = t4i + e + 1;
                if (t > s) {
                    d = fmul(d, av[e]);
                    dm[t * C1 + s] = d;
                }
            }
        }
    }
    __syncthreads();
    // Gram on the tensor cores: the (m16, n8) tiles of the lower triangle,
    // spread over the warps; each tile's chain runs over d_k in 8-wide blocks
    constexpr int MT = C / 16, NTILE = MT * (MT + 1);  // tile (m, q) with q <= 2m+1
    for (int tile = warp; tile < NTILE; tile += nwarps) {
        int m = 0;
        while ((m + 1) * (m + 2) <= tile) ++m;
        const int q = tile - m * (m + 1);
        const int r0 = m * 16, n0 = q * 8;
        float acc[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.f;
#pragma unroll 4
        for (int kb = 0; kb < DK / 8; ++kb) {
            const int k0 = kb * 8;
            const float a0 = kx[(r0 + g) * KXS + k0 + t4], a1 = kx[(r0 + g + 8) * KXS + k0 + t4];
            const float a2 = kx[(r0 + g) * KXS + k0 + t4 + 4], a3 = kx[(r0 + g + 8) * KXS + k0 + t4 + 4];
            const float b0 = kx[(n0 + g) * KXS + k0 + t4], b1 = kx[(n0 + g) * KXS + k0 + t4 + 4];
            if (k_exact) {
                const uint32_t ah[4] = {__float_as_uint(a0), __float_as_uint(a1), __float_as_uint(a2),
                                        __float_as_uint(a3)};
                const uint32_t bh[2] = {__float_as_uint(b0), __float_as_uint(b1)};
                mma_tf32(acc[kb & 3], ah, bh);
            } else {
                uint32_t ah[4], al[4], bh[2], bl[2];
                tf32_split(a0, ah[0], al[0]); tf32_split(a1, ah[1], al[1]);
                tf32_split(a2, ah[2], al[2]); tf32_split(a3, ah[3], al[3]);
                tf32_split(b0, bh[0], bl[0]); tf32_split(b1, bh[1], bl[1]);
                mma_tf32(acc[0], al, bh);
                mma_tf32(acc[1], ah, bl);
                mma_tf32(acc[2], ah, bh);
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int tau = r0 + g + (c >> 1) * 8, sig = n0 + 2 * t4 + (c & 1);
            const float G = k_exact ? fadd(fadd(acc[0][c], acc[1][c]), fadd(acc[2][c], acc[3][c]))
                                    : fadd(fadd(acc[0][c], acc[1][c]), acc[2][c]);
            if (sig < tau) cc[tau * CCS + sig] = fmul(dm[(tau + 1) * C1 + (sig + 1)], G);
        }
    }
    for (int t = threadIdx.x; t < C; t += blockDim.x) d0[t] = dm[(t + 1) * C1];  // D[t][0], t = 1..C
    if (dCout != nullptr)
        for (int s = threadIdx.x; s <= C; s += blockDim.x) dCout[s] = dm[C * C1 + s];
    __syncthreads();
    float* stage = dm;  // [16][STS]: the block's accumulators
    for (int b = 0; b < C / 16; ++b) {
        const int t0 = 16 * b;
        // init + tensor-core part: warp w owns column tiles w, w + nw, ... (each
        // tile all u0 or all w columns); its tiles share the split c fragment
        {
            constexpr int NTW = (NCOL / 8 + 7) / 8;  // tiles per warp with 8 warps
            float init[NTW][4], plh[NTW][4], phl[NTW][4], phh[NTW][4];
            const float* xb[NTW];
            int xs[NTW];
#pragma unroll
            for (int q = 0; q < NTW; ++q) {
                const int nt = warp + nwarps * q;
                const int n0 = nt * 8;
                const bool is_u = n0 < DV;
                xb[q] = is_u ? vx + n0 : kx + (n0 - DV);
                xs[q] = is_u ? VXS : KXS;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    plh[q][c] = phl[q][c] = phh[q][c] = 0.f;
                    const int tau = t0 + g + (c >> 1) * 8, cl = 2 * t4 + (c & 1);
                    init[q][c] = nt >= NCOL / 8 ? 0.f
                                 : is_u ? xb[q][tau * xs[q] + cl] : fmul(d0[tau], xb[q][tau * xs[q] + cl]);
                }
            }
            for (int kb = 0; kb < 2 * b; ++kb) {
                const int s0 = kb * 8;
                uint32_t ah[4], al[4];
                tf32_split(-cc[(t0 + g) * CCS + s0 + t4], ah[0], al[0]);
                tf32_split(-cc[(t0 + g + 8) * CCS + s0 + t4], ah[1], al[1]);
                tf32_split(-cc[(t0 + g) * CCS + s0 + t4 + 4], ah[2], al[2]);
                tf32_split(-cc[(t0 + g + 8) * CCS + s0 + t4 + 4], ah[3], al[3]);
#pragma unroll
                for (int q = 0; q < NTW; ++q) {
                    if (warp + nwarps * q < NCOL / 8) {
                        uint32_t bh[2], bl[2];
                        tf32_split(xb[q][(s0 + t4) * xs[q] + g], bh[0], bl[0]);
                        tf32_split(xb[q][(s0 + t4 + 4) * xs[q] + g], bh[1], bl[1]);
                        mma_tf32(plh[q], al, bh);
                        mma_tf32(phl[q], ah, bl);
                        mma_tf32(phh[q], ah, bh);
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < NTW; ++q) {
                const int nt = warp + nwarps * q;
                if (nt < NCOL / 8) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float acc = b == 0 ? init[q][c]
                                                 : fadd(init[q][c], fadd(fadd(plh[q][c], phl[q][c]), phh[q][c]));
                        stage[(g + (c >> 1) * 8) * STS + nt * 8 + 2 * t4 + (c & 1)] = acc;
                    }
                }
            }
        }
        __syncthreads();
        // in-block part: one column per thread, sequential over the block's 16 tokens
        for (int col = threadIdx.x; col < NCOL; col += blockDim.x) {
            float xb[16];
#pragma unroll
            for (int tr = 0; tr < 16; ++tr) {
                float acc = stage[tr * STS + col];
#pragma unroll
                for (int sr = 0; sr < tr; ++sr) acc = ffma(-cc[(t0 + tr) * CCS + t0 + sr], xb[sr], acc);
                xb[tr] = fmul(bs[t0 + tr], acc);
            }
#pragma unroll
            for (int tr = 0; tr < 16; ++tr) {
                const int tau = t0 + tr;
                if (col < DV) {
                    vx[tau * VXS + col] = xb[tr];
                    uout[tau * ldu + col] = xb[tr];
                } else {
                    kx[tau * KXS + (col - DV)] = xb[tr];
                    wout[tau * ldw + (col - DV)] = xb[tr];
                }
            }
        }
        __syncthreads();
    }
}

template <int DK, int DV, int C>
struct PrepSmem {
    using PL = PrepLayout<DK, DV, C>;
    static constexpr int KX_OFF = 0;
    static constexpr int VX_OFF = KX_OFF + C * PL::KXS;
    static constexpr int CC_OFF = VX_OFF + C * PL::VXS;
    static constexpr int DM_OFF = CC_OFF + C * PL::CCS;
    static constexpr int D0_OFF = DM_OFF + ((PL::DM + 3) / 4) * 4;
    static constexpr int AB_OFF = D0_OFF + C + 4;
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
    using PL = PrepLayout<DK, DV, C>;
    if (__ldg(err)) return;
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    float* kx = sm + Sm::KX_OFF;
    float* vx = sm + Sm::VX_OFF;
    float* cc = sm + Sm::CC_OFF;
    float* dm = sm + Sm::DM_OFF;
    float* d0 = sm + Sm::D0_OFF;
    float* as = sm + Sm::AB_OFF;
    float* bs = as + C;

    const int task = blockIdx.x;
    const int h = task % H, g = task / H;
    const int n = find_seq(fco, N, g);
    const int64_t tok0 = (int64_t)__ldg(cu + n) + (int64_t)(g - __ldg(fco + n)) * C;
    for (int t = threadIdx.x; t < C; t += blockDim.x) {
        cp_async4(as + t, alpha + (tok0 + t) * H + h);
        cp_async4(bs + t, beta + (tok0 + t) * H + h);
    }
    if (in_bf16) {
        // raw bf16 rows [k | v] of the chunk land in the c / decay buffers
        // (unused until the Gram), all copies in flight at once; then widen
        static_assert(Sm::DM_OFF + ((PL::DM + 3) / 4) * 4 - Sm::CC_OFF >= C * (DK + DV) / 2, "raw staging fits");
        unsigned char* raw = reinterpret_cast<unsigned char*>(cc);
        constexpr int PK = DK / 8, PV = DV / 8;  // 16-byte pieces per row
        for (int e = threadIdx.x; e < C * (PK + PV); e += blockDim.x) {
            const int t = e / (PK + PV), pc = e % (PK + PV);
            const int64_t row = (tok0 + t) * H + h;
            const uint16_t* src = pc < PK ? reinterpret_cast<const uint16_t*>(k) + row * DK + pc * 8
                                          : reinterpret_cast<const uint16_t*>(v) + row * DV + (pc - PK) * 8;
            cp_async16(raw + (size_t)e * 16, src);
        }
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
        for (int e = threadIdx.x; e < C * (PK + PV); e += blockDim.x) {
            const int t = e / (PK + PV), pc = e % (PK + PV);
            float x[8];
            lds8_raw(raw + (size_t)e * 16, 0, 1, x);
            float* d = pc < PK ? kx + t * PL::KXS + pc * 8 : vx + t * PL::VXS + (pc - PK) * 8;
            *reinterpret_cast<float4*>(d) = make_float4(x[0], x[1], x[2], x[3]);
            *reinterpret_cast<float4*>(d + 4) = make_float4(x[4], x[5], x[6], x[7]);
        }
    } else {
        stage_rows<DK>(kx, PL::KXS, k, tok0, C, H, h, in_bf16, IdxIdentity());
        stage_rows<DV>(vx, PL::VXS, v, tok0, C, H, h, in_bf16, IdxIdentity());
        cp_async_commit();
        cp_async_wait_all();
    }
    __syncthreads();
    chunk_prep<DK, DV, C>(kx, vx, as, bs, cc, dm, d0, in_bf16, w_ws + (int64_t)task * C * DK, DK,
                          u_ws + (int64_t)task * C * DV, DV, dC_ws + (int64_t)task * Cf::DCS);
}

template <int DK, int DV, int C>
struct ChainSmem {
    using T = TcCfg<DK, DV, C>;
    static constexpr int WRS = DK + 4;                       // raw w row stride (conflict-free conversion reads)
    static constexpr int WLO_OFF = 0;                        // canonical w lo | hi (adjacent)
    static constexpr int WHI_OFF = WLO_OFF + T::W_FLOATS;
    static constexpr int KLO_OFF = WHI_OFF + T::W_FLOATS;    // canonical k^T lo | hi (adjacent), then S' staging
    static constexpr int KHI_OFF = KLO_OFF + T::K_FLOATS;
    static constexpr int WRAW_OFF = KLO_OFF + T::K_REGION;   // [C][WRS] the next chunk's w, in flight
    static constexpr int US_OFF = WRAW_OFF + C * WRS;        // [C][DV] u0
    static constexpr int DC_OFF = US_OFF + C * DV;           // [C+4] D[C][.]
    static constexpr int BAR_OFF = DC_OFF + ChunkCfg<DK, DV, C>::DCS;  // mbarrier (8 bytes) + TMEM base
    // at least 120 KB, so that one CTA fits per SM: each allocates all 512 TMEM columns
    static constexpr size_t USED = sizeof(float) * (BAR_OFF + 4);
    static constexpr size_t BYTES = USED > 120 * 1024 ? USED : 120 * 1024;
    static_assert(BYTES <= 232448, "fits the 227 KB of shared memory a CTA can have");
    static_assert(BAR_OFF % 2 == 0 && WRAW_OFF % 4 == 0 && US_OFF % 4 == 0, "alignment");
};

// Boundary states: one CTA per (sequence, head), serial over the sequence's
// full chunks, on the tensor cores (tcgen05; the state stays in TMEM and in
// registers between chunks).  Writes chunk_states[so[n] + c] for
// c = 0..floor(L/C).  Thread 0 issues the MMAs; while they run, warps 1..7
// move data: during phase 1 they store the previous chunk's S' rows, write this
// chunk's k^T (loaded into registers one chunk ahead) and start the next
// chunk's w and k loads; during phase 2 they convert the next chunk's w into
// the split operands and start its u0 and decay copies.  An MMA completion
// wait that times out records GDN_ERR_TIMEOUT in *err and ends the CTA; the
// kernels after it then write nothing.
//
// progress (when non-null) publishes, for the pair, how many of its chunk
// states are in global memory: after state c is written (and fenced),
// progress[nh] = c + 1, with release semantics.  With withhold != 0 nothing is
// published (the failure-detection test hook).
template <int DK, int DV, int C>
__device__ __forceinline__ void chain_run(const void* __restrict__ k, const float* __restrict__ state_in,
                                          const int32_t* __restrict__ cu, const int32_t* __restrict__ fco,
                                          const int32_t* __restrict__ so, int32_t* err, int H, int in_bf16,
                                          const float* __restrict__ w_ws, const float* __restrict__ u_ws,
                                          const float* __restrict__ dC_ws, float* states, int nh,
                                          int32_t* progress, int withhold, float* sm)
{
    using Cf = ChunkCfg<DK, DV, C>;
    using Sm = ChainSmem<DK, DV, C>;
    using T = TcCfg<DK, DV, C>;
    constexpr int NP = T::THREADS - 32;  // data-moving threads: warps 1..7
    float* Whi = sm + Sm::WHI_OFF;
    float* Wlo = sm + Sm::WLO_OFF;
    float* Khi = sm + Sm::KHI_OFF;
    float* Klo = sm + Sm::KLO_OFF;
    float* wraw = sm + Sm::WRAW_OFF;
    float* us = sm + Sm::US_OFF;
    float* dCs = sm + Sm::DC_OFF;
    uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + Sm::BAR_OFF);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Sm::BAR_OFF + 2);

    const int h = nh % H, n = nh / H;
    const int seq0 = __ldg(cu + n);
    const int nfull = (__ldg(cu + n + 1) - seq0) / C;
    const int64_t slot0 = __ldg(so + n);
    const int64_t g0 = __ldg(fco + n);
    const bool mover = threadIdx.x >= 32;
    const int pt = threadIdx.x - 32;  // index among the data-moving threads
    auto state_dst = [&](int c) { return states + ((slot0 + c) * H + h) * (int64_t)DV * DK; };
    auto movers_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(NP) : "memory"); };
    auto publish = [&](int count) {  // after a fence and a barrier over the writers
        if (progress != nullptr && !withhold) st_release_gpu(progress + nh, count);
    };

    auto fetch_w = [&](int c, int tid, int nthr) {  // raw w of chunk c -> wraw
        const float* src = w_ws + ((g0 + c) * H + h) * (int64_t)C * DK;
        for (int e = tid; e < C * DK / 4; e += nthr) {
            const int t = e / (DK / 4), j4 = (e % (DK / 4)) * 4;
            cp_async16(wraw + t * Sm::WRS + j4, src + t * DK + j4);
        }
        cp_async_commit();
    };
    auto fetch_u = [&](int c, int tid, int nthr) {  // u0 and D[C][.] of chunk c
        const int64_t task = (g0 + c) * H + h;
        const float* usrc = u_ws + task * C * DV;
        for (int e = tid; e < C * DV / 4; e += nthr) cp_async16(us + 4 * e, usrc + 4 * e);
        for (int e = tid; e < Cf::DCS / 4; e += nthr) cp_async16(dCs + 4 * e, dC_ws + task * Cf::DCS + 4 * e);
        cp_async_commit();
    };

    if (threadIdx.x == 0) mbar_init(mbar, 1);
    if (threadIdx.x < 32) tmem_alloc(tslot, T::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;
    const TcThread<DK> th(tbase);

    float SR[DK / 2];
    tc_load_state<DK, DV, C>(SR, th, state_in != nullptr ? state_in + ((int64_t)n * H + h) * DV * DK : nullptr,
                             state_dst(0));
    if (nfull > 0) {  // chunk 0's operands, by every thread
        fetch_w(0, threadIdx.x, T::THREADS);
        fetch_u(0, threadIdx.x, T::THREADS);
        tc_stage_kT<DK, DV, C>(k, (int64_t)seq0, H, h, in_bf16, Khi, Klo);
        cp_async_wait_all();
        __syncthreads();
        tc_stage_w<DK, DV, C>(wraw, Sm::WRS, Whi, Wlo, threadIdx.x, T::THREADS);
    }
    __threadfence();  // state 0 (written by every thread above) is visible ...
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) publish(1);  // ... before it is published

    KPrefetch<DK, DV, C, NP> kpre;
    uint32_t parity = 0;
    bool ok = true;
    for (int c = 0; c < nfull; ++c) {
        const bool more = c + 1 < nfull;
        if (threadIdx.x == 0) tc_issue_phase1<DK, DV, C>(tbase, Wlo, mbar);
        if (mover) {
            if (c > 0) {
                tc_store_rows<DK, DV>(Klo, state_dst(c), nullptr, pt, NP);  // S' of chunk c-1, staged in Klo
                __threadfence();
                movers_sync();
                if (pt == 0) publish(c + 1);
                kpre.store(Khi, Klo, in_bf16, pt);                            // k^T of chunk c
                fence_async_smem();
            }
            if (more) {
                fetch_w(c + 1, pt, NP);
                kpre.load(k, (int64_t)seq0 + (int64_t)(c + 1) * C, H, h, in_bf16, pt);
                cp_async_wait_1();  // u0 and decays of chunk c (w of chunk c+1 may still be in flight)
            } else {
                cp_async_wait_all();
            }
        }
        ok = tc_wait(mbar, parity);
        if (!ok) break;
        const float d0 = tc_epilogue_e<DK, DV, C>(th, us, DV, dCs);
        if (threadIdx.x == 0) tc_issue_phase2<DK, DV, C>(tbase, Klo, in_bf16, mbar);
        if (mover && more) {  // phase 1 is done with w: the next chunk's w goes in while phase 2 runs
            cp_async_wait_all();
            movers_sync();
            tc_stage_w<DK, DV, C>(wraw, Sm::WRS, Whi, Wlo, pt, NP);
            fence_async_smem();
            fetch_u(c + 1, pt, NP);
        }
        ok = tc_wait(mbar, parity);
        if (!ok) break;
        tc_epilogue_S<DK, DV, C>(SR, th, d0, in_bf16, Klo);
    }
    if (ok && nfull > 0 && mover) {
        tc_store_rows<DK, DV>(Klo, state_dst(nfull), nullptr, pt, NP);
        __threadfence();
    }
    if (!ok && threadIdx.x == 0) record_error(err, GDN_ERR_TIMEOUT);
    cp_async_wait_all();
    tc_fence_before();
    __syncthreads();
    if (ok && nfull > 0 && threadIdx.x == 0) publish(nfull + 1);
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(tbase, T::TMEM_COLS);
    }
}

template <int DK, int DV, int C>
__global__ void __launch_bounds__(256, 1)
k_chain(const void* __restrict__ k, const float* __restrict__ state_in, const int32_t* __restrict__ cu,
        const int32_t* __restrict__ fco, const int32_t* __restrict__ so, int32_t* err, int N, int H, int in_bf16,
        const float* __restrict__ w_ws, const float* __restrict__ u_ws, const float* __restrict__ dC_ws,
        float* __restrict__ states)
{
    if (*reinterpret_cast<volatile int32_t*>(err)) return;
    extern __shared__ float4 smem_f4[];
    chain_run<DK, DV, C>(k, state_in, cu, fco, so, err, H, in_bf16, w_ws, u_ws, dC_ws, states, blockIdx.x, nullptr,
                         0, reinterpret_cast<float*>(smem_f4));
}

// ------------------------------------------------------------------ fused chain + P_tok
template <int DK, int DV, int C>
struct FusedSmem {
    static constexpr size_t TOK = ((TokCfg<DK, DV, C>::SMEM + 15) / 16) * 16;  // one P_tok task
    static constexpr size_t BYTES = ChainSmem<DK, DV, C>::BYTES > 2 * TOK ? ChainSmem<DK, DV, C>::BYTES : 2 * TOK;
    static constexpr bool OK = TokCfg<DK, DV, C>::THREADS == 128;  // two P_tok tasks per 256-thread CTA
};

// Boundary chain and intra-chunk recurrence in one cooperative launch, for
// batches with fewer (sequence, head) pairs than SMs.  CTA b < N*H runs the
// chain of pair b (publishing progress[b] as its states land), then joins the
// others as a P_tok worker.  Workers take P_tok tasks from one queue in
// chunk-major order (task t -> chunk c with cumc[c] <= t < cumc[c+1],
// sequence order[t - cumc[c]], the sequences sorted by chunk count), two
// tasks per CTA at a time (one per 128-thread half), each after its boundary
// state is published.  Every CTA is resident (cooperative launch), and chains
// wait on nothing, so every wait ends.  A wait gives up after wait_limit
// clocks (kWaitLimit, about a second, in normal operation), records
// GDN_ERR_TIMEOUT in *err and ends its half; withhold != 0 (the test hook)
// makes the chains publish nothing, so every wait runs out.
template <int DK, int DV, int C>
__global__ void __launch_bounds__(256, 1)
k_chain_tok(const void* __restrict__ q, const void* __restrict__ k, const void* __restrict__ v,
            const float* __restrict__ alpha, const float* __restrict__ beta, const float* __restrict__ state_in,
            const int32_t* __restrict__ cu, const int32_t* __restrict__ fco, const int32_t* __restrict__ so,
            int32_t* err, int N, int H, int in_bf16, int out_bf16, const float* __restrict__ w_ws,
            const float* __restrict__ u_ws, const float* __restrict__ dC_ws, float* states, void* __restrict__ o,
            float* __restrict__ cacheR, int32_t* progress, int32_t* tok_next, const int32_t* __restrict__ order,
            const int32_t* __restrict__ cumc, int maxc, int withhold, long long wait_limit)
{
    using Fs = FusedSmem<DK, DV, C>;
    static_assert(Fs::OK, "d_v = 128: two 128-thread P_tok tasks per CTA");
    volatile int32_t* verr = err;
    if (*verr) return;
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    if ((int)blockIdx.x < N * H) {
        chain_run<DK, DV, C>(k, state_in, cu, fco, so, err, H, in_bf16, w_ws, u_ws, dC_ws, states, blockIdx.x,
                             progress, withhold, sm);
        __syncthreads();
    }
    const int half = threadIdx.x >> 7, tid = threadIdx.x & 127;
    float* tsm = sm + half * (Fs::TOK / 4);
    const HalfSync hs{2 + half};
    __shared__ int qslot[2], go[2];
    const int ntask = __ldg(cumc + maxc);
    // Thread 0 of a half claims its next queue slot one task ahead, so the
    // atomic's round trip overlaps the current task.
    int next = tid == 0 ? atomicAdd(tok_next, 1) : 0;
    for (;;) {
        if (tid == 0) qslot[half] = next;
        hs();
        const int qi = qslot[half];
        if (qi >= ntask * H) break;
        const int t = qi / H, h = qi % H;
        int lo = 0, hi = maxc;  // cumc[0] = 0 <= t < cumc[maxc]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(cumc + mid) <= t) lo = mid; else hi = mid;
        }
        const int c = lo, n = __ldg(order + t - __ldg(cumc + c));
        if (tid == 0) {  // one thread waits and decides for the half
            next = atomicAdd(tok_next, 1);
            // The acquire load orders this half's later state loads after the
            // chain's release (through the barrier below): no fence needed.
            const bool ready = wait_at_least(progress + (int64_t)n * H + h, c + 1, wait_limit);
            if (!ready) record_error(err, GDN_ERR_TIMEOUT);
            go[half] = ready && *verr == 0;
        }
        hs();
        if (!go[half]) break;
        const int seq0 = __ldg(cu + n);
        tok_task<DK, DV, C, true>(q, k, v, alpha, beta, n, c, h, H, seq0, __ldg(cu + n + 1) - seq0,
                                  (int64_t)__ldg(so + n) + c, in_bf16, out_bf16, states, o, cacheR, tsm, tid, hs);
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

}  // namespace gdn
