// k_pchunk.cuh -- chunk-boundary update P_chunk: k_prep, k_chain, k_cache_fill (sm_100a).
#pragma once

#include "k_ptok.cuh"

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

// ---------------------------------------------------------------- tensor-core P_chunk part 2
// The two contractions of the boundary update on the tensor cores
// (mma.sync m16n8k8, tf32 operands, fp32 accumulate), with every fp32
// operand x split into hi = tf32(x) and lo = tf32(x - hi):
//   phase 1: E[i][t] = sum_j S[i][j] w_t[j]; per 8-wide block of j, in
//            ascending order: E += S_lo*w_hi, E += S_hi*w_lo, E += S_hi*w_hi;
//            then e_t[i] = D[C][t] * (u0_t[i] - E[i][t]).
//   phase 2: S'[i][j] = D[C][0]*S[i][j] + sum_t e_t[i] k_t[j]; accumulator
//            starts at D[C][0]*S[i][j], then per 8-token block, ascending:
//            S' += e_lo*k_hi, S' += e_hi*k_lo, S' += e_hi*k_hi.  When k is
//            exactly tf32 (bf16 inputs), k_lo = 0 and that product is skipped.
// The prefill chain and the decode resync run these same functions, so the
// same operands give the same bits.  A CTA has 4 warps on a tile of RTB rows
// (RTB = 16 or 32): warp w owns m16 tile w % MT and every WG-th n8 tile.
template <int DK, int RTB, int C>
struct MmaAdv {
    static constexpr int MT = RTB / 16;             // m16 row tiles
    static constexpr int WG = 4 / MT;               // warps sharing a row tile
    static constexpr int NT1 = C / 8, NT2 = DK / 8;
    static constexpr int P1 = (NT1 + WG - 1) / WG;  // phase-1 n8 tiles per warp
    static constexpr int P2 = (NT2 + WG - 1) / WG;  // phase-2 n8 tiles per warp
    static constexpr int KS = DK + 4;               // S and w row stride (floats)
    static constexpr int ES = C + 4;                // e and k^T row stride (floats)
    static constexpr int THREADS = 128;
    static_assert(RTB == 16 || RTB == 32, "row tile");
};

// Phase 1 (warps 0..3): es[i*ES + t] = e_t[i] for the RTB rows of the tile.
template <int DK, int RTB, int C>
__device__ __forceinline__ void mma_phase1(const float* Ss, const float* ws, const float* us, int ldu,
                                           const float* dCs, float* es)
{
    using M = MmaAdv<DK, RTB, C>;
    constexpr int KS = M::KS, ES = M::ES;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    if (warp >= 4) return;
    const int mt = warp % M::MT, wg = warp / M::MT, r0 = mt * 16;
    // one accumulator per split product (independent tensor-core chains)
    float alh[M::P1][4], ahl[M::P1][4], ahh[M::P1][4];
#pragma unroll
    for (int q = 0; q < M::P1; ++q)
#pragma unroll
        for (int c = 0; c < 4; ++c) alh[q][c] = ahl[q][c] = ahh[q][c] = 0.f;
#pragma unroll 2
    for (int kb = 0; kb < DK / 8; ++kb) {
        const int k0 = kb * 8;
        uint32_t ah[4], al[4];
        tf32_split(Ss[(r0 + g) * KS + k0 + t], ah[0], al[0]);
        tf32_split(Ss[(r0 + g + 8) * KS + k0 + t], ah[1], al[1]);
        tf32_split(Ss[(r0 + g) * KS + k0 + t + 4], ah[2], al[2]);
        tf32_split(Ss[(r0 + g + 8) * KS + k0 + t + 4], ah[3], al[3]);
#pragma unroll
        for (int q = 0; q < M::P1; ++q) {
            const int nt = wg + M::WG * q;
            if (nt < M::NT1) {
                uint32_t bh[2], bl[2];
                tf32_split(ws[(nt * 8 + g) * KS + k0 + t], bh[0], bl[0]);
                tf32_split(ws[(nt * 8 + g) * KS + k0 + t + 4], bh[1], bl[1]);
                mma_tf32(alh[q], al, bh);
                mma_tf32(ahl[q], ah, bl);
                mma_tf32(ahh[q], ah, bh);
            }
        }
    }
#pragma unroll
    for (int q = 0; q < M::P1; ++q) {
        const int nt = wg + M::WG * q;
        if (nt < M::NT1) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int i = r0 + g + (c >> 1) * 8, tau = nt * 8 + 2 * t + (c & 1);
                const float E = fadd(fadd(alh[q][c], ahl[q][c]), ahh[q][c]);
                es[i * ES + tau] = fmul(dCs[tau + 1], fsub(us[tau * ldu + i], E));
            }
        }
    }
}

// Phase 2 (warps 0..3): Sreg (this lane's entries of the tile in the phase-2
// accumulator layout) <- S'.  The new rows also go to Ss and, when non-null,
// to dst1 / dst2 (global, row stride DK).  k_exact: k values are exact tf32.
template <int DK, int RTB, int C, bool K_EXACT>
__device__ __forceinline__ void mma_phase2_t(float (&Sreg)[MmaAdv<DK, RTB, C>::P2][4], float* Ss, const float* es,
                                             const float* kT, float d0, float* dst1, float* dst2)
{
    using M = MmaAdv<DK, RTB, C>;
    constexpr int KS = M::KS, ES = M::ES;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    if (warp >= 4) return;
    const int mt = warp % M::MT, wg = warp / M::MT, r0 = mt * 16;
    constexpr int NHL = K_EXACT ? 1 : M::P2;  // the k_lo product is absent when k is exact tf32
    float alh[M::P2][4], ahl[NHL][4], ahh[M::P2][4];
#pragma unroll
    for (int q = 0; q < M::P2; ++q)
#pragma unroll
        for (int c = 0; c < 4; ++c) alh[q][c] = ahh[q][c] = 0.f;
#pragma unroll
    for (int q = 0; q < NHL; ++q)
#pragma unroll
        for (int c = 0; c < 4; ++c) ahl[q][c] = 0.f;
#pragma unroll 1
    for (int kb = 0; kb < C / 8; ++kb) {
        const int k0 = kb * 8;
        uint32_t ah[4], al[4];
        tf32_split(es[(r0 + g) * ES + k0 + t], ah[0], al[0]);
        tf32_split(es[(r0 + g + 8) * ES + k0 + t], ah[1], al[1]);
        tf32_split(es[(r0 + g) * ES + k0 + t + 4], ah[2], al[2]);
        tf32_split(es[(r0 + g + 8) * ES + k0 + t + 4], ah[3], al[3]);
#pragma unroll
        for (int q = 0; q < M::P2; ++q) {
            const int nt = wg + M::WG * q;
            if (nt < M::NT2) {
                const float b0 = kT[(nt * 8 + g) * ES + k0 + t], b1 = kT[(nt * 8 + g) * ES + k0 + t + 4];
                if constexpr (K_EXACT) {
                    const uint32_t b[2] = {__float_as_uint(b0), __float_as_uint(b1)};
                    mma_tf32(alh[q], al, b);
                    mma_tf32(ahh[q], ah, b);
                } else {
                    uint32_t bh[2], bl[2];
                    tf32_split(b0, bh[0], bl[0]);
                    tf32_split(b1, bh[1], bl[1]);
                    mma_tf32(alh[q], al, bh);
                    mma_tf32(ahl[q], ah, bl);
                    mma_tf32(ahh[q], ah, bh);
                }
            }
        }
    }
#pragma unroll
    for (int q = 0; q < M::P2; ++q) {
        const int nt = wg + M::WG * q;
        if (nt < M::NT2) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float x = fadd(fmul(d0, Sreg[q][c]), alh[q][c]);
                if constexpr (!K_EXACT) x = fadd(x, ahl[q][c]);
                Sreg[q][c] = fadd(x, ahh[q][c]);
            }
#pragma unroll
            for (int hrow = 0; hrow < 2; ++hrow) {
                const int i = r0 + g + hrow * 8, j = nt * 8 + 2 * t;
                const float2 x = make_float2(Sreg[q][2 * hrow], Sreg[q][2 * hrow + 1]);
                *reinterpret_cast<float2*>(Ss + i * KS + j) = x;
                if (dst1 != nullptr) *reinterpret_cast<float2*>(dst1 + (int64_t)i * DK + j) = x;
                if (dst2 != nullptr) *reinterpret_cast<float2*>(dst2 + (int64_t)i * DK + j) = x;
            }
        }
    }
}

template <int DK, int RTB, int C>
__device__ __forceinline__ void mma_phase2(float (&Sreg)[MmaAdv<DK, RTB, C>::P2][4], float* Ss, const float* es,
                                           const float* kT, float d0, int k_exact, float* dst1, float* dst2)
{
    if (k_exact) mma_phase2_t<DK, RTB, C, true>(Sreg, Ss, es, kT, d0, dst1, dst2);
    else mma_phase2_t<DK, RTB, C, false>(Sreg, Ss, es, kT, d0, dst1, dst2);
}

// Load the RTB rows at src (global, row stride DK) into Ss and this lane's
// phase-2 registers (warps 0..3).  Ends with a barrier.
template <int DK, int RTB, int C>
__device__ __forceinline__ void mma_load_state(float (&Sreg)[MmaAdv<DK, RTB, C>::P2][4], float* Ss, const float* src)
{
    using M = MmaAdv<DK, RTB, C>;
    for (int e = threadIdx.x; e < RTB * (DK / 4); e += blockDim.x) {
        const int i = e / (DK / 4), j4 = (e % (DK / 4)) * 4;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (src != nullptr) x = *reinterpret_cast<const float4*>(src + (int64_t)i * DK + j4);
        *reinterpret_cast<float4*>(Ss + i * M::KS + j4) = x;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    if (warp < 4) {
        const int mt = warp % M::MT, wg = warp / M::MT, r0 = mt * 16;
#pragma unroll
        for (int q = 0; q < M::P2; ++q) {
            const int nt = wg + M::WG * q;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                Sreg[q][c] = nt < M::NT2 ? Ss[(r0 + g + (c >> 1) * 8) * M::KS + nt * 8 + 2 * t + (c & 1)] : 0.f;
        }
    }
}

// k of C tokens (rows of a [T, H, DK] input from token tok0, head h) -> kT
// [DK][ES] fp32 (transposed; token index fastest across threads, so the
// scattered stores hit consecutive banks).
template <int DK, int C>
__device__ __forceinline__ void stage_kT(float* kT, const void* k, int64_t tok0, int H, int h, int bf16)
{
    constexpr int ES = C + 4;
    for (int e = threadIdx.x; e < C * (DK / 8); e += blockDim.x) {
        const int tau = e % C, j8 = (e / C) * 8;
        float x[8];
        load8(k, ((tok0 + tau) * H + h) * (int64_t)DK + j8, bf16, x);
#pragma unroll
        for (int m = 0; m < 8; ++m) kT[(j8 + m) * ES + tau] = x[m];
    }
}

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
    using Cf = ChunkCfg<DK, DV, C>;
    using M = MmaAdv<DK, Cf::RTB, C>;
    static constexpr int SS_OFF = 0;                              // [RTB][KS] fp32 S
    static constexpr int WS_OFF = SS_OFF + Cf::RTB * M::KS;       // [C][KS] w
    static constexpr int ES_OFF = WS_OFF + C * M::KS;             // [RTB][ES] e
    static constexpr int KT_OFF = ES_OFF + Cf::RTB * M::ES;       // [DK][ES] k^T
    static constexpr int US_OFF = KT_OFF + DK * M::ES;            // [C][RTB] u0 rows of the tile
    static constexpr int DC_OFF = US_OFF + C * Cf::RTB;           // [C+4] D[C][.]
    static constexpr size_t BYTES = sizeof(float) * (DC_OFF + Cf::DCS);
};

// Boundary states: one CTA (4 warps) per (sequence, head, row tile), serial
// over the sequence's full chunks; the tile's state stays in registers.
// Writes chunk_states[so[n] + c] for c = 0..floor(L/C).  The next chunk's w,
// u0 and decays arrive by cp.async during phase 2.
template <int DK, int DV, int C>
__global__ void __launch_bounds__(128)
k_chain(const void* __restrict__ k, const float* __restrict__ state_in, const int32_t* __restrict__ cu,
        const int32_t* __restrict__ fco, const int32_t* __restrict__ so, const int32_t* __restrict__ err,
        int N, int H, int in_bf16, const float* __restrict__ w_ws, const float* __restrict__ u_ws,
        const float* __restrict__ dC_ws, float* __restrict__ states)
{
    using Cf = ChunkCfg<DK, DV, C>;
    using Sm = ChainSmem<DK, DV, C>;
    using M = MmaAdv<DK, Cf::RTB, C>;
    constexpr int KS = M::KS, RTB = Cf::RTB;
    if (__ldg(err)) return;
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    float* Ss = sm + Sm::SS_OFF;
    float* ws = sm + Sm::WS_OFF;
    float* es = sm + Sm::ES_OFF;
    float* kT = sm + Sm::KT_OFF;
    float* us = sm + Sm::US_OFF;
    float* dCs = sm + Sm::DC_OFF;

    const int r = blockIdx.x % Cf::NTB;
    const int nh = blockIdx.x / Cf::NTB;
    const int h = nh % H, n = nh / H;
    const int seq0 = __ldg(cu + n);
    const int nfull = (__ldg(cu + n + 1) - seq0) / C;
    const int64_t slot0 = __ldg(so + n);
    const int64_t g0 = __ldg(fco + n);
    const int64_t row0 = (int64_t)r * RTB;

    auto fetch = [&](int c) {
        const int64_t task = (g0 + c) * H + h;
        const float* wsrc = w_ws + task * C * DK;
        for (int e = threadIdx.x; e < C * (DK / 4); e += blockDim.x) {
            const int t = e / (DK / 4), j4 = (e % (DK / 4)) * 4;
            cp_async16(ws + t * KS + j4, wsrc + t * DK + j4);
        }
        const float* usrc = u_ws + task * C * DV + row0;
        for (int e = threadIdx.x; e < C * (RTB / 4); e += blockDim.x) {
            const int t = e / (RTB / 4), i4 = (e % (RTB / 4)) * 4;
            cp_async16(us + t * RTB + i4, usrc + t * DV + i4);
        }
        for (int e = threadIdx.x; e < Cf::DCS / 4; e += blockDim.x)
            cp_async16(dCs + 4 * e, dC_ws + task * Cf::DCS + 4 * e);
        cp_async_commit();
    };

    float Sreg[M::P2][4];
    mma_load_state<DK, RTB, C>(Sreg, Ss,
                               state_in != nullptr ? state_in + (((int64_t)n * H + h) * DV + row0) * DK : nullptr);
    for (int e = threadIdx.x; e < RTB * (DK / 4); e += blockDim.x) {
        const int i = e / (DK / 4), j4 = (e % (DK / 4)) * 4;
        *reinterpret_cast<float4*>(states + ((slot0 * H + h) * DV + row0 + i) * DK + j4) =
            *reinterpret_cast<const float4*>(Ss + i * KS + j4);
    }
    if (nfull > 0) {
        fetch(0);
        stage_kT<DK, C>(kT, k, (int64_t)seq0, H, h, in_bf16);
    }
    for (int c = 0; c < nfull; ++c) {
        cp_async_wait_all();
        __syncthreads();  // w/u0/D and k of chunk c are in smem; Ss is current
        mma_phase1<DK, RTB, C>(Ss, ws, us, RTB, dCs, es);
        const float d0 = dCs[0];
        __syncthreads();  // e complete; w, u0 and D may be overwritten
        if (c + 1 < nfull) fetch(c + 1);
        // bf16 inputs: the next chunk's k (raw 16-byte pieces) is loaded into
        // registers now and written to smem after phase 2, so the load latency
        // overlaps the tensor-core work
        constexpr int ITEMS = C * (DK / 8), NPRE = (ITEMS + M::THREADS - 1) / M::THREADS;
        uint4 kpre[NPRE];
        const int64_t tok1 = (int64_t)seq0 + (int64_t)(c + 1) * C;
        if (c + 1 < nfull && in_bf16) {
#pragma unroll
            for (int i = 0; i < NPRE; ++i) {
                const int e = threadIdx.x + i * M::THREADS;
                if (e < ITEMS) {
                    const int tau = e % C, j8 = (e / C) * 8;
                    kpre[i] = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(k) +
                                                                   ((tok1 + tau) * H + h) * (int64_t)DK + j8));
                }
            }
        }
        mma_phase2<DK, RTB, C>(Sreg, Ss, es, kT, d0, in_bf16,
                               states + (((slot0 + c + 1) * H + h) * DV + row0) * DK, nullptr);
        if (c + 1 < nfull) {
            __syncthreads();  // phase 2 is done with k
            if (in_bf16) {
#pragma unroll
                for (int i = 0; i < NPRE; ++i) {
                    const int e = threadIdx.x + i * M::THREADS;
                    if (e < ITEMS) {
                        const int tau = e % C, j8 = (e / C) * 8;
                        const uint32_t w4[4] = {kpre[i].x, kpre[i].y, kpre[i].z, kpre[i].w};
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            kT[(j8 + 2 * m) * M::ES + tau] = __uint_as_float(w4[m] << 16);
                            kT[(j8 + 2 * m + 1) * M::ES + tau] = __uint_as_float(w4[m] & 0xffff0000u);
                        }
                    }
                }
            } else {
                stage_kT<DK, C>(kT, k, tok1, H, h, in_bf16);
            }
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

}  // namespace gdn
