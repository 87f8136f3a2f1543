// k_prep.cuh -- P_chunk part 1, the chunk-local precompute (sm_100a).
//
// For one chunk of C tokens (1-indexed t inside the chunk) it produces the
// operands of the boundary update (k_tc.cuh):
//   D[s][s] = 1, D[t][s] = D[t-1][s] * alpha_t          decay products (fp32 chains)
//   G[t][s] = k_t . k_s (s < t)                          Gram, on the tensor cores (mma.sync)
//   A[t][s] = beta_t * (D[t][s] * G[t][s])  (s < t)      L = I + A, unit lower triangular
//   T       = L^{-1}                                     blocked: 16 x 16 diagonal blocks by
//                                                        substitution, off-diagonal blocks by
//                                                        tensor-core products (mma.sync)
//   u0      = T diag(beta) V,  w = T diag(gamma) K,  gamma_t = beta_t * D[t][0]
//                                                        tcgen05, transposed (below)
// so that w_t = beta_t (D[t][0] k_t - sum_{s<t} c_ts w_s) and u0_t likewise
// from v_t, with c_ts = D[t][s] G[t][s]: the forward substitution of the
// chunkwise form, solved through the inverse of its triangular matrix.  The
// inverse keeps the sequential part to 16-token blocks of one 64-wide matrix
// and puts the products with the 2 d-wide right-hand side into dense
// tensor-core products, and [u0 | w] never has to be read back.
//
// Tensor-core products are "3xTF32": an fp32 operand x is split as
// hi = tf32_rna(x), lo = tf32_rna(x - hi).  An operand that is exact in tf32
// (k and v from bf16 inputs) has lo = 0 and its products are skipped.
//   mma.sync (Gram, T's off-diagonal blocks): lo*hi, hi*lo and hi*hi
//   accumulate over k blocks of 8 in ascending order, each in its own fp32
//   accumulator, and the result is (lo*hi + hi*lo) + hi*hi; the exact Gram is
//   hi*hi alone, accumulated in four chains by k block mod 4 and summed
//   (a0 + a1) + (a2 + a3).
//   tcgen05 ([u0 | w]): u0^T = V^T (T diag(beta))^T, w^T = K^T (T diag(gamma))^T
//   with M = 128 feature rows (rows past d are zero), A = V^T or K^T in tensor
//   memory (a feature per lane, a token per column) and B = the scaled T, one
//   16-token row block n per MMA group (N = 16, K = 16 (n + 1): T is lower
//   triangular), K-major in shared memory.  Each row block has one fp32
//   accumulator, fed in this order over K blocks of 8 ascending: V.T_lo, then
//   V.T_hi for bf16 inputs; V_hi.T_lo, V_lo.T_hi, V_hi.T_hi otherwise.
// The prefill (k_prep), the backward (k_bprep) and the decode resync call the
// same function, so all produce the same bits.
#pragma once

#include "k_ptok.cuh"
#include "k_tc.cuh"

namespace gdn {

template <int DK, int DV, int C>
struct PrepCfg {
    static_assert(DK == DV && DK <= 128 && C % 16 == 0 && C <= 64, "prep shapes");
    static constexpr int NB = C / 16;          // 16-token blocks
    static constexpr int MS = C + 4;           // row stride of A, T and the decays (floats)
    static constexpr int SS = 16 + 4;          // row stride of the 16 x 16 scratch blocks
    static constexpr int NCOL = DV + DK;       // columns of [u0 | w]
    // raw input rows, in the input dtype, padded by 16 bytes per row: the row
    // stride is 4 words mod 32, which keeps the fragment reads conflict-free
    __host__ __device__ static constexpr int krb(int bf16) { return DK * (bf16 ? 2 : 4) + 16; }
    __host__ __device__ static constexpr int vrb(int bf16) { return DV * (bf16 ? 2 : 4) + 16; }
    // B operands of the [u0 | w] products: row block n of the scaled T as a
    // canonical K-major tile [16 rows t][16 (n + 1) columns s] (8-row groups
    // 512 (n + 1) bytes apart, 4-column groups 128 bytes apart); the hi tiles,
    // then the lo tiles.  They take the A and M scratch, dead by then.
    __host__ __device__ static constexpr int bt_off(int n) { return 128 * n * (n + 1); }  // floats
    static constexpr int BT_FL = 128 * NB * (NB + 1);   // one split half
    // float offsets of the scratch that follows the raw rows: TD | A | M | small | barrier
    static constexpr int TD_FL = (C + 1) * MS;
    static constexpr int A_FL = C * MS;
    static constexpr int M_FL0 = (NB > 1 ? NB - 1 : 1) * 16 * SS;
    static constexpr int M_FL = 2 * BT_FL - A_FL > M_FL0 ? 2 * BT_FL - A_FL : M_FL0;
    static constexpr int SMALL_FL = 5 * (C + 4);  // d0, dC, alpha, beta, gamma
    static constexpr int BAR_FL = 4;              // mbarrier (8 bytes) and the TMEM base
    static constexpr int SCRATCH_FL = TD_FL + A_FL + M_FL + SMALL_FL + BAR_FL;
    static_assert(MS % 4 == 0 && M_FL % 4 == 0 && SMALL_FL % 2 == 0, "16-byte tiles, 8-byte barrier");
    __host__ __device__ static constexpr size_t raw_bytes(int bf16) { return (size_t)C * (krb(bf16) + vrb(bf16)); }
    __host__ __device__ static constexpr size_t bytes(int bf16) { return raw_bytes(bf16) + 4 * (size_t)SCRATCH_FL; }
    // tensor memory: accumulator [0, C), A operand hi [C, 2C), lo [2C, 3C) (fp32 inputs)
    static constexpr uint32_t ACC = 0, AHI = C, ALO = 2 * C;
    __host__ __device__ static constexpr uint32_t tmem_cols(int bf16)
    {
        return (bf16 ? 2 : 3) * C <= 32 ? 32 : (bf16 ? 2 : 3) * C <= 64 ? 64 : (bf16 ? 2 : 3) * C <= 128 ? 128 : 256;
    }
    // kind::tf32, fp32 accumulate, A and B K-major, M = 128, N = 16
    static constexpr uint32_t IDESC = (1u << 4) | (2u << 7) | (2u << 10) | ((16u >> 3) << 17) | ((128u >> 4) << 24);
};

// The shared-memory pieces chunk_prep works on.
struct PrepBufs {
    const unsigned char* kr;  // [C] raw k rows (input dtype), stride krb
    const unsigned char* vr;  // [C] raw v rows, stride vrb
    float* TD;                // [C+1][MS]: decays, then T
    float* A;                 // [C][MS]
    float* M;                 // [NB-1][16][SS]
    float* BT;                // the B tiles of the products (over A and M)
    float* d0;                // [C]: D[t][0], t = 1..C
    float* dC;                // [C+1]: D[C][s]
    const float* as;          // [C] alpha
    const float* bs;          // [C] beta
    float* gam;               // [C] gamma_t = beta_t * D[t][0]
    uint64_t* mbar;           // MMA completion barrier (prep_tc_open)
    uint32_t* tslot;          // TMEM base (prep_tc_open)
};

template <int DK, int DV, int C>
__device__ __forceinline__ PrepBufs prep_bufs(unsigned char* base, int bf16)
{
    using P = PrepCfg<DK, DV, C>;
    PrepBufs b;
    b.kr = base;
    b.vr = base + (size_t)C * P::krb(bf16);
    float* f = reinterpret_cast<float*>(base + P::raw_bytes(bf16));
    b.TD = f;
    b.A = f + P::TD_FL;
    b.M = b.A + P::A_FL;
    b.BT = b.A;
    b.d0 = b.M + P::M_FL;
    b.dC = b.d0 + (C + 4);
    float* as = b.dC + (C + 4);
    b.as = as;
    b.bs = as + (C + 4);
    b.gam = as + 2 * (C + 4);
    b.mbar = reinterpret_cast<uint64_t*>(as + 3 * (C + 4));
    b.tslot = reinterpret_cast<uint32_t*>(as + 3 * (C + 4) + 2);
    return b;
}

template <bool BF>
__device__ __forceinline__ float ld_raw(const unsigned char* rowp, int col)
{
    if constexpr (BF) return __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(rowp)[col] << 16);
    else return reinterpret_cast<const float*>(rowp)[col];
}

// 3xTF32 products of one m16n8 tile over k blocks [kb0, kb1): fa(kb, i) gives
// the A fragment's fp32 value i (0..3), fb(kb, i) the B fragment's (0..1).
template <typename FA, typename FB>
__device__ __forceinline__ void mma3_tile(float (&lh)[4], float (&hl)[4], float (&hh)[4], int kb0, int kb1, FA fa,
                                          FB fb)
{
    for (int kb = kb0; kb < kb1; ++kb) {
        uint32_t ah[4], al[4], bh[2], bl[2];
#pragma unroll
        for (int i = 0; i < 4; ++i) tf32_split(fa(kb, i), ah[i], al[i]);
#pragma unroll
        for (int i = 0; i < 2; ++i) tf32_split(fb(kb, i), bh[i], bl[i]);
        mma_tf32(lh, al, bh);
        mma_tf32(hl, ah, bl);
        mma_tf32(hh, ah, bh);
    }
}

__device__ __forceinline__ float sum3(float lh, float hl, float hh) { return fadd(fadd(lh, hl), hh); }

// P_chunk part 1 of one chunk by one CTA of 256 threads.  BF: the raw rows
// are bf16 (else fp32).  The caller has staged the raw k, v rows and the gates
// (b.as, b.bs) and synchronised; tbase holds PrepCfg::tmem_cols(BF) free TMEM
// columns, mbar is an initialised mbarrier whose next phase has the given
// parity (flipped on each use).  Writes u0 -> uout[t * ldu + i], w ->
// wout[t * ldw + j] (any address space) and, when dCout is non-null,
// D[C][s] -> dCout[s].  Returns false on every thread if an MMA completion
// wait timed out (the outputs are then incomplete).  Ends with a barrier,
// after which the TMEM columns are free again.
template <int DK, int DV, int C, bool BF>
__device__ __forceinline__ bool chunk_prep(const PrepBufs& b, uint32_t tbase, uint64_t* mbar, uint32_t& parity,
                                           float* uout, int ldu, float* wout, int ldw, float* dCout)
{
    using P = PrepCfg<DK, DV, C>;
    constexpr int MS = P::MS, SS = P::SS, NB = P::NB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
    const int nwarps = blockDim.x >> 5;
    constexpr int krb = P::krb(BF), vrb = P::vrb(BF);
    float* TD = b.TD;
    if constexpr (BF) {
        // Re-lay each 8-element block of the raw k rows as (0,4,1,5,2,6,3,7):
        // 32-bit word j then holds elements j and j + 4, the pair one lane of
        // an m16n8k8 fragment takes, so one load serves both.
        unsigned char* kr = const_cast<unsigned char*>(b.kr);
        for (int e = threadIdx.x; e < C * (DK / 8); e += blockDim.x) {
            uint4* p = reinterpret_cast<uint4*>(kr + (size_t)(e / (DK / 8)) * krb + 16 * (e % (DK / 8)));
            const uint4 x = *p;
            *p = make_uint4(__byte_perm(x.x, x.z, 0x5410), __byte_perm(x.x, x.z, 0x7632),
                            __byte_perm(x.y, x.w, 0x5410), __byte_perm(x.y, x.w, 0x7632));
        }
    }
    // decay products: column s is the chain D[t][s] = D[t-1][s] * alpha_t.  The
    // loop over t is unrolled with s as a predicate, so the alpha loads are
    // independent of the chain and issue ahead of it.
    for (int s = threadIdx.x; s <= C; s += blockDim.x) {
        float d = 1.0f;
        TD[s * MS + s] = d;
#pragma unroll
        for (int t = 1; t <= C; ++t) {
            const float a = b.as[t - 1];
            if (t > s) {
                d = fmul(d, a);
                TD[t * MS + s] = d;
            }
        }
    }
    __syncthreads();
    // Gram on the tensor cores, by 16 x 16 blocks (m, p <= m) of the lower
    // triangle, each two (m16, n8) tiles that share the A fragment;
    // A[t][s] = beta_t * (D[t][s] * G[t][s]) (1-indexed t, s)
    {
        constexpr int MT = C / 16, NBLK = MT * (MT + 1) / 2;
        for (int blk = warp; blk < NBLK; blk += nwarps) {
            int m = 0;
            while ((m + 1) * (m + 2) / 2 <= blk) ++m;
            const int p = blk - m * (m + 1) / 2;
            const int r0 = m * 16;
            const unsigned char* ra = b.kr + (size_t)(r0 + g) * krb;
            const unsigned char* rb = b.kr + (size_t)(r0 + g + 8) * krb;
            float acc[2][4][4];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int u = 0; u < 4; ++u) acc[h][u][0] = acc[h][u][1] = acc[h][u][2] = acc[h][u][3] = 0.f;
#pragma unroll 4
            for (int kb = 0; kb < DK / 8; ++kb) {
                const int k0 = kb * 8;
                if constexpr (BF) {  // re-laid rows: word k0/2 + t4 holds elements k0 + t4 and k0 + t4 + 4
                    const uint32_t xa = reinterpret_cast<const uint32_t*>(ra)[k0 / 2 + t4];
                    const uint32_t xb = reinterpret_cast<const uint32_t*>(rb)[k0 / 2 + t4];
                    const uint32_t ah[4] = {xa << 16, xb << 16, xa & 0xffff0000u, xb & 0xffff0000u};
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t xn = reinterpret_cast<const uint32_t*>(
                            b.kr + (size_t)(16 * p + 8 * h + g) * krb)[k0 / 2 + t4];
                        const uint32_t bh[2] = {xn << 16, xn & 0xffff0000u};
                        mma_tf32(acc[h][kb & 3], ah, bh);
                    }
                } else {
                    uint32_t ah[4], al[4];
                    tf32_split(ld_raw<BF>(ra, k0 + t4), ah[0], al[0]);
                    tf32_split(ld_raw<BF>(rb, k0 + t4), ah[1], al[1]);
                    tf32_split(ld_raw<BF>(ra, k0 + t4 + 4), ah[2], al[2]);
                    tf32_split(ld_raw<BF>(rb, k0 + t4 + 4), ah[3], al[3]);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const unsigned char* rn = b.kr + (size_t)(16 * p + 8 * h + g) * krb;
                        uint32_t bh[2], bl[2];
                        tf32_split(ld_raw<BF>(rn, k0 + t4), bh[0], bl[0]);
                        tf32_split(ld_raw<BF>(rn, k0 + t4 + 4), bh[1], bl[1]);
                        mma_tf32(acc[h][0], al, bh);
                        mma_tf32(acc[h][1], ah, bl);
                        mma_tf32(acc[h][2], ah, bh);
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int tau = r0 + g + (c >> 1) * 8, sig = 16 * p + 8 * h + 2 * t4 + (c & 1);
                    const float G = BF ? fadd(fadd(acc[h][0][c], acc[h][1][c]), fadd(acc[h][2][c], acc[h][3][c]))
                                       : fadd(fadd(acc[h][0][c], acc[h][1][c]), acc[h][2][c]);
                    if (sig < tau) b.A[tau * MS + sig] = fmul(b.bs[tau], fmul(TD[(tau + 1) * MS + (sig + 1)], G));
                }
        }
    }
    for (int t = threadIdx.x; t < C; t += blockDim.x) {  // D[t][0] and gamma_t = beta_t * D[t][0], t = 1..C
        b.d0[t] = TD[(t + 1) * MS];
        b.gam[t] = fmul(b.bs[t], TD[(t + 1) * MS]);
    }
    for (int s = threadIdx.x; s <= C; s += blockDim.x) {
        b.dC[s] = TD[C * MS + s];
        if (dCout != nullptr) dCout[s] = TD[C * MS + s];
    }
    __syncthreads();  // the decays are consumed: TD now takes T
    // diagonal blocks of T by substitution: thread i owns column i of its
    // block; for s ascending, T[s][i] is final, then acc_t = fma(-A[t][s], T[s][i], acc_t)
    // for every later row t of the block (acc_t starts at 0; T[i][i] = 1)
    if (threadIdx.x < C) {
        const int i = threadIdx.x, i0 = i & ~15, ri = i & 15;
        float acc[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) acc[t] = 0.f;
#pragma unroll
        for (int s = 0; s < 15; ++s) {
            const float x = s == ri ? 1.0f : acc[s];
#pragma unroll
            for (int t = s + 1; t < 16; ++t) {
                const float a = b.A[(i0 + t) * MS + i0 + s];
                acc[t] = s >= ri ? ffma(-a, x, acc[t]) : acc[t];
            }
        }
#pragma unroll
        for (int t = 0; t < 16; ++t) TD[(i0 + t) * MS + i] = t > ri ? acc[t] : (t == ri ? 1.0f : 0.0f);
    }
    __syncthreads();
    // off-diagonal blocks, by distance d below the diagonal: warp j computes
    // block (i = j + d, j) as  M = A[i-rows][16j, 16i) T[16j, 16i)[j-cols], then
    // T_ij = -(T_ii M), both on the tensor cores (3xTF32)
    for (int d = 1; d < NB; ++d) {
        const int j = warp;
        const int i = j + d;
        float* Mj = b.M + j * 16 * SS;
        if (i < NB) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int n0 = 16 * j + 8 * nt;
                float lh[4] = {0.f, 0.f, 0.f, 0.f}, hl[4] = {0.f, 0.f, 0.f, 0.f}, hh[4] = {0.f, 0.f, 0.f, 0.f};
                mma3_tile(lh, hl, hh, 2 * j, 2 * i,
                          [&](int kb, int u) {
                              return b.A[(16 * i + g + (u & 1) * 8) * MS + 8 * kb + t4 + (u >> 1) * 4];
                          },
                          [&](int kb, int u) { return TD[(8 * kb + t4 + u * 4) * MS + n0 + g]; });
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    Mj[(g + (c >> 1) * 8) * SS + 8 * nt + 2 * t4 + (c & 1)] = sum3(lh[c], hl[c], hh[c]);
            }
        }
        __syncwarp();
        if (i < NB) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                float lh[4] = {0.f, 0.f, 0.f, 0.f}, hl[4] = {0.f, 0.f, 0.f, 0.f}, hh[4] = {0.f, 0.f, 0.f, 0.f};
                mma3_tile(lh, hl, hh, 0, 2,
                          [&](int kb, int u) {
                              return TD[(16 * i + g + (u & 1) * 8) * MS + 16 * i + 8 * kb + t4 + (u >> 1) * 4];
                          },
                          [&](int kb, int u) { return Mj[(8 * kb + t4 + u * 4) * SS + 8 * nt + g]; });
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    TD[(16 * i + g + (c >> 1) * 8) * MS + 16 * j + 8 * nt + 2 * t4 + (c & 1)] =
                        -sum3(lh[c], hl[c], hh[c]);
            }
        }
        __syncthreads();
    }
    // [u0 | w] on tcgen05, one product per pass: u0^T = V^T (T diag(beta))^T,
    // then w^T = K^T (T diag(gamma))^T, gamma_s = beta_s * D[s][0].
    {
        const int q = warp & 3, hf = warp >> 2;        // TMEM lane quarter, half of the token columns
        const int f = 32 * q + lane;                   // feature row of this thread
        const uint32_t lane_base = tbase + ((uint32_t)(32 * q) << 16);
        constexpr int CH = C / 2;
        // a k row's element f sits at 8 (f / 8) + 2 (f % 4) + (f % 8) / 4 once re-laid (bf16)
        const int fk = BF ? 8 * (f >> 3) + 2 * (f & 3) + ((f >> 2) & 1) : f;
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
            const float* scale = pass ? b.gam : b.bs;
            // B tiles: element (t, s) of row block n = (T[t][s] * scale[s]) split, 16-byte items
            // of 4 columns; 8 consecutive items fill one 128-byte core matrix
            constexpr int ITEMS = 32 * NB * (NB + 1);
            for (int e = threadIdx.x; e < ITEMS; e += blockDim.x) {
                int n = 0;
                while (32 * (n + 1) * (n + 2) <= e) ++n;
                const int l = e - 32 * n * (n + 1), r8 = l & 7, kg = 4 * (n + 1);
                const int k4 = (l >> 3) % kg, rg = (l >> 3) / kg;
                const int t = 16 * n + 8 * rg + r8;
                const float4 x = *reinterpret_cast<const float4*>(TD + t * MS + 4 * k4);
                uint32_t h[4], lo[4];
                tf32_split(fmul(x.x, scale[4 * k4]), h[0], lo[0]);
                tf32_split(fmul(x.y, scale[4 * k4 + 1]), h[1], lo[1]);
                tf32_split(fmul(x.z, scale[4 * k4 + 2]), h[2], lo[2]);
                tf32_split(fmul(x.w, scale[4 * k4 + 3]), h[3], lo[3]);
                const int off = P::bt_off(n) + rg * 128 * (n + 1) + k4 * 32 + r8 * 4;
                *reinterpret_cast<uint4*>(b.BT + off) = make_uint4(h[0], h[1], h[2], h[3]);
                *reinterpret_cast<uint4*>(b.BT + P::BT_FL + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            // A operand: row f of V^T (or K^T), tokens hf * C/2 .. + C/2, into TMEM
            const unsigned char* src = pass ? b.kr : b.vr;
            const int rs = pass ? krb : vrb, col = pass ? fk : f;
#pragma unroll
            for (int c8 = 0; c8 < CH / 8; ++c8) {
                uint32_t hi8[8], lo8[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float x = f < DK ? ld_raw<BF>(src + (size_t)(hf * CH + 8 * c8 + m) * rs, col) : 0.0f;
                    if constexpr (BF) hi8[m] = __float_as_uint(x);
                    else tf32_split(x, hi8[m], lo8[m]);
                }
                tmem_st8(lane_base + P::AHI + hf * CH + 8 * c8, hi8);
                if constexpr (!BF) tmem_st8(lane_base + P::ALO + hf * CH + 8 * c8, lo8);
            }
            tmem_wait_st();
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            if (threadIdx.x == 0) {
                tc_fence_after();
                const uint32_t bt = smem_u32(b.BT);
#pragma unroll 1
                for (int n = 0; n < NB; ++n) {
                    const uint32_t d = tbase + P::ACC + 16 * n, bh = bt + 4u * P::bt_off(n), bl = bh + 4u * P::BT_FL;
                    const uint32_t sbo = 512u * (n + 1);
                    const int nk = 2 * n + 2;
                    if constexpr (BF) {
                        for (int kb = 0; kb < nk; ++kb)
                            mma_tf32_ts(d, tbase + P::AHI + 8 * kb, smem_desc(bl + 256u * kb, 128u, sbo), P::IDESC, kb > 0);
                        for (int kb = 0; kb < nk; ++kb)
                            mma_tf32_ts(d, tbase + P::AHI + 8 * kb, smem_desc(bh + 256u * kb, 128u, sbo), P::IDESC, 1);
                    } else {
                        for (int kb = 0; kb < nk; ++kb)
                            mma_tf32_ts(d, tbase + P::AHI + 8 * kb, smem_desc(bl + 256u * kb, 128u, sbo), P::IDESC, kb > 0);
                        for (int kb = 0; kb < nk; ++kb)
                            mma_tf32_ts(d, tbase + P::ALO + 8 * kb, smem_desc(bh + 256u * kb, 128u, sbo), P::IDESC, 1);
                        for (int kb = 0; kb < nk; ++kb)
                            mma_tf32_ts(d, tbase + P::AHI + 8 * kb, smem_desc(bh + 256u * kb, 128u, sbo), P::IDESC, 1);
                    }
                }
                mma_commit(mbar);
            }
            if (!tc_wait(mbar, parity)) return false;
            // epilogue: accumulator column t of lane f is u0_t[f] (w_t[f])
            float* out = pass ? wout : uout;
            const int ld = pass ? ldw : ldu;
#pragma unroll
            for (int c8 = 0; c8 < CH / 8; ++c8) {
                float x[8];
                tmem_ld8(lane_base + P::ACC + hf * CH + 8 * c8, x);
                if (f < DK) {
#pragma unroll
                    for (int m = 0; m < 8; ++m) out[(int64_t)(hf * CH + 8 * c8 + m) * ld + f] = x[m];
                }
            }
            tc_fence_before();
            __syncthreads();  // the accumulator, A and the B tiles are free again
            tc_fence_after();
        }
    }
    return true;
}

// Stage one chunk's raw k, v rows (token rows tok0.., head h of [T, H, D]
// tensors, or of the decode buffers with H = 1) and gates into the layout of
// prep_bufs, by cp.async; the caller commits, waits and synchronises.
template <int DK, int DV, int C>
__device__ __forceinline__ void prep_stage(unsigned char* base, const void* k, const void* v, const float* alpha,
                                           const float* beta, int64_t tok0, int H, int h, int bf16)
{
    using P = PrepCfg<DK, DV, C>;
    const PrepBufs b = prep_bufs<DK, DV, C>(base, bf16);
    const int esz = bf16 ? 2 : 4;
    const int pk = DK * esz / 16, pv = DV * esz / 16;  // 16-byte pieces per row
    unsigned char* kr = const_cast<unsigned char*>(b.kr);
    unsigned char* vr = const_cast<unsigned char*>(b.vr);
    for (int e = threadIdx.x; e < C * (pk + pv); e += blockDim.x) {
        const int t = e / (pk + pv), pc = e % (pk + pv);
        const int64_t row = (tok0 + t) * H + h;
        if (pc < pk)
            cp_async16(kr + (size_t)t * P::krb(bf16) + 16 * pc, reinterpret_cast<const char*>(k) + row * DK * esz + 16 * pc);
        else
            cp_async16(vr + (size_t)t * P::vrb(bf16) + 16 * (pc - pk),
                       reinterpret_cast<const char*>(v) + row * DV * esz + 16 * (pc - pk));
    }
    float* as = const_cast<float*>(b.as);
    float* bs = const_cast<float*>(b.bs);
    for (int t = threadIdx.x; t < C; t += blockDim.x) {
        cp_async4(as + t, alpha + (tok0 + t) * H + h);
        cp_async4(bs + t, beta + (tok0 + t) * H + h);
    }
}

// chunk_prep with the input dtype chosen at run time (both forms inlined).
template <int DK, int DV, int C>
__device__ __forceinline__ bool chunk_prep_any(const PrepBufs& b, int bf16, uint32_t tbase, uint64_t* mbar,
                                               uint32_t& parity, float* uout, int ldu, float* wout, int ldw,
                                               float* dCout)
{
    if (bf16) return chunk_prep<DK, DV, C, true>(b, tbase, mbar, parity, uout, ldu, wout, ldw, dCout);
    return chunk_prep<DK, DV, C, false>(b, tbase, mbar, parity, uout, ldu, wout, ldw, dCout);
}

// For a kernel that runs chunk_prep alone: its mbarrier (in b) initialised
// and PrepCfg::tmem_cols(BF) TMEM columns allocated; returns their base.
template <int DK, int DV, int C, bool BF>
__device__ __forceinline__ uint32_t prep_tc_open(const PrepBufs& b)
{
    if (threadIdx.x == 0) mbar_init(b.mbar, 1);
    if (threadIdx.x < 32) tmem_alloc(b.tslot, PrepCfg<DK, DV, C>::tmem_cols(BF));
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return *b.tslot;
}

// The TMEM of prep_tc_open freed (every thread calls it, after chunk_prep).
template <int DK, int DV, int C, bool BF>
__device__ __forceinline__ void prep_tc_close(uint32_t tbase)
{
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(tbase, PrepCfg<DK, DV, C>::tmem_cols(BF));
    }
}

// P_chunk part 1 for every full chunk: one CTA per (full chunk, head).  BF:
// bf16 inputs (else fp32), fixed at compile time.
template <int DK, int DV, int C, bool BF>
__global__ void __launch_bounds__(256, 3)
k_prep(const void* __restrict__ k, const void* __restrict__ v, const float* __restrict__ alpha,
       const float* __restrict__ beta, const int32_t* __restrict__ cu, const int32_t* __restrict__ fco,
       int32_t* err, int N, int H,
       float* __restrict__ w_ws, float* __restrict__ u_ws, float* __restrict__ dC_ws)
{
    constexpr int in_bf16 = BF;
    if (*reinterpret_cast<volatile const int32_t*>(err)) return;
    extern __shared__ float4 smem_f4[];
    unsigned char* base = reinterpret_cast<unsigned char*>(smem_f4);
    const int task = blockIdx.x;
    const int h = task % H, g = task / H;
    const int n = find_seq(fco, N, g);
    const int64_t tok0 = (int64_t)__ldg(cu + n) + (int64_t)(g - __ldg(fco + n)) * C;
    prep_stage<DK, DV, C>(base, k, v, alpha, beta, tok0, H, h, in_bf16);
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    const PrepBufs b = prep_bufs<DK, DV, C>(base, in_bf16);
    const uint32_t tbase = prep_tc_open<DK, DV, C, BF>(b);
    uint32_t parity = 0;
    if (!chunk_prep<DK, DV, C, BF>(b, tbase, b.mbar, parity, u_ws + (int64_t)task * C * DV, DV,
                                   w_ws + (int64_t)task * C * DK, DK, dC_ws + (int64_t)task * (C + 4)) &&
        threadIdx.x == 0)
        record_error(err, GDN_ERR_TIMEOUT);
    prep_tc_close<DK, DV, C, BF>(tbase);
}

}  // namespace gdn
