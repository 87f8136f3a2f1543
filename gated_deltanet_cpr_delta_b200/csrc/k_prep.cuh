// k_prep.cuh -- P_chunk part 1, the chunk-local precompute (sm_100a).
//
// For one chunk of C tokens (1-indexed t inside the chunk) it produces the
// operands of the boundary update (k_tc.cuh):
//   D[s][s] = 1, D[t][s] = D[t-1][s] * alpha_t          decay products (fp32 chains)
//   G[t][s] = k_t . k_s (s < t)                          Gram, on the tensor cores
//   A[t][s] = beta_t * (D[t][s] * G[t][s])  (s < t)      L = I + A, unit lower triangular
//   T       = L^{-1}                                     blocked: 16 x 16 diagonal blocks by
//                                                        substitution, off-diagonal blocks by
//                                                        tensor-core products
//   u0      = T diag(beta) V,  w = T diag(gamma) K,  gamma_t = beta_t * D[t][0]
//                                                        tensor cores
// so that w_t = beta_t (D[t][0] k_t - sum_{s<t} c_ts w_s) and u0_t likewise
// from v_t, with c_ts = D[t][s] G[t][s]: the forward substitution of the
// chunkwise form, solved through the inverse of its triangular matrix.  The
// inverse keeps the sequential part to 16-token blocks of one 64-wide matrix
// and puts the products with the 2 d-wide right-hand side into dense
// tensor-core products, and [u0 | w] never has to be read back.
//
// Tensor-core products are "3xTF32": an fp32 operand x is split as
// hi = tf32_rna(x), lo = tf32_rna(x - hi); lo*hi, hi*lo and hi*hi accumulate
// over k blocks of 8 in ascending order, each in its own fp32 accumulator,
// and the result is (lo*hi + hi*lo) + hi*hi.  An operand that is exact in tf32
// (k and v from bf16 inputs) has lo = 0 and its products are skipped: the
// Gram is then hi*hi alone, accumulated in four chains by k block mod 4 and
// summed (a0 + a1) + (a2 + a3), and [u0 | w] is (lo*V) + (hi*V).  The prefill (k_prep) and the decode
// resync call the same function, so both produce the same bits.
#pragma once

#include "k_ptok.cuh"

namespace gdn {

template <int DK, int DV, int C>
struct PrepCfg {
    static constexpr int NB = C / 16;          // 16-token blocks
    static constexpr int MS = C + 4;           // row stride of A, T and the decays (floats)
    static constexpr int NCOL = DV + DK;       // columns of [u0 | w]
    // raw input rows, in the input dtype, padded by 16 bytes per row: the row
    // stride is 4 words mod 32, which keeps the fragment reads conflict-free
    __host__ __device__ static constexpr int krb(int bf16) { return DK * (bf16 ? 2 : 4) + 16; }
    __host__ __device__ static constexpr int vrb(int bf16) { return DV * (bf16 ? 2 : 4) + 16; }
    // float offsets of the scratch that follows the raw rows: A | TD | small.
    // The off-diagonal steps of T keep their 16 x 16 intermediates M_j in A's
    // unused upper triangle (block (j, NB-1)).
    static constexpr int A_FL = C * MS;
    static constexpr int TD_FL = (C + 1) * MS;
    static constexpr int SMALL_FL = 5 * (C + 4);  // d0, dC, alpha, beta, gamma
    static constexpr int SCRATCH_FL = A_FL + TD_FL + SMALL_FL;
    // bf16 v rows that fit in A's region go there once A is dead (chunk_prep
    // stages them after T is complete): v is needed only by the products
    __host__ __device__ static constexpr bool v_in_a(int bf16) { return bf16 && C * vrb(bf16) <= 4 * A_FL; }
    __host__ __device__ static constexpr size_t raw_bytes(int bf16)
    {
        return (size_t)C * krb(bf16) + (v_in_a(bf16) ? 0 : (size_t)C * vrb(bf16));
    }
    __host__ __device__ static constexpr size_t bytes(int bf16) { return raw_bytes(bf16) + 4 * (size_t)SCRATCH_FL; }
    // CTAs of 256 threads that the shared memory allows per SM (4 needs at most 64 registers a thread)
    __host__ __device__ static constexpr int ctas_per_sm(int bf16) { return bytes(bf16) + 1024 <= 233472 / 4 ? 4 : 3; }
};

// Where a chunk's v rows come from: rows (tok0 + t) * H + h of a [T, H, DV]
// tensor for t < len, zero rows after.
struct VSrc {
    const void* v;
    int64_t tok0;
    int H, h, len;
};

template <int DV, int C, bool BF>
__device__ __forceinline__ void stage_v_rows(const VSrc& s, unsigned char* vr, int vrb, int tid, int nthr)
{
    constexpr int esz = BF ? 2 : 4, pv = DV * esz / 16;  // 16-byte pieces per row
    for (int e = tid; e < C * pv; e += nthr) {
        const int t = e / pv, pc = e % pv;
        unsigned char* dst = vr + (size_t)t * vrb + 16 * pc;
        if (t < s.len)
            cp_async16(dst, reinterpret_cast<const char*>(s.v) + ((s.tok0 + t) * s.H + s.h) * DV * esz + 16 * pc);
        else
            *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
}

// The shared-memory pieces chunk_prep works on.
struct PrepBufs {
    const unsigned char* kr;  // [C] raw k rows (input dtype), stride krb
    const unsigned char* vr;  // [C] raw v rows, stride vrb
    float* A;                 // [C][MS]
    float* TD;                // [C+1][MS]: decays, then T
    float* M;                 // M_j at M + 16 j MS, row stride MS (A's upper triangle)
    float* d0;                // [C]: D[t][0], t = 1..C
    float* dC;                // [C+1]: D[C][s]
    const float* as;          // [C] alpha
    const float* bs;          // [C] beta
    float* gam;               // [C] gamma_t = beta_t * D[t][0]
};

template <int DK, int DV, int C>
__device__ __forceinline__ PrepBufs prep_bufs(unsigned char* base, int bf16)
{
    using P = PrepCfg<DK, DV, C>;
    PrepBufs b;
    b.kr = base;
    float* f = reinterpret_cast<float*>(base + P::raw_bytes(bf16));
    b.vr = P::v_in_a(bf16) ? reinterpret_cast<unsigned char*>(f) : base + (size_t)C * P::krb(bf16);
    b.A = f;
    b.TD = f + P::A_FL;
    b.M = f + 16 * (P::NB - 1);
    b.d0 = b.TD + P::TD_FL;
    b.dC = b.d0 + (C + 4);
    float* as = b.dC + (C + 4);
    b.as = as;
    b.bs = as + (C + 4);
    b.gam = as + 2 * (C + 4);
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

// P_chunk part 1 of one chunk by one CTA of 256 threads.
// BF: the raw rows are bf16 (else fp32).  The caller has staged the raw k
// rows, the v rows unless PrepCfg::v_in_a (then chunk_prep stages them from
// vs once T is complete) and the gates (b.as, b.bs), and synchronised.
// Writes u0 -> uout[t * ldu + i], w -> wout[t * ldw + j] (any address space)
// and, when dCout is non-null, D[C][s] -> dCout[s].  Ends with a barrier.
template <int DK, int DV, int C, bool BF>
__device__ __forceinline__ void chunk_prep(const PrepBufs& b, const VSrc& vs, float* uout, int ldu, float* wout,
                                           int ldw, float* dCout)
{
    using P = PrepCfg<DK, DV, C>;
    constexpr int MS = P::MS, NB = P::NB;
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
    // off-diagonal blocks, by distance d below the diagonal: block (i = j + d, j)
    // is M = A[i-rows][16j, 16i) T[16j, 16i)[j-cols], then T_ij = -(T_ii M),
    // both on the tensor cores (3xTF32).  Each 8-column half nt of the block
    // needs only its own columns of M, so warp 2 j + nt computes it alone.
    for (int d = 1; d < NB; ++d) {
        const int j = warp >> 1, nt = warp & 1;
        const int i = j + d;
        float* Mj = b.M + j * 16 * MS;
        if (i < NB) {
            {
                const int n0 = 16 * j + 8 * nt;
                float lh[4] = {0.f, 0.f, 0.f, 0.f}, hl[4] = {0.f, 0.f, 0.f, 0.f}, hh[4] = {0.f, 0.f, 0.f, 0.f};
                mma3_tile(lh, hl, hh, 2 * j, 2 * i,
                          [&](int kb, int u) {
                              return b.A[(16 * i + g + (u & 1) * 8) * MS + 8 * kb + t4 + (u >> 1) * 4];
                          },
                          [&](int kb, int u) { return TD[(8 * kb + t4 + u * 4) * MS + n0 + g]; });
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    Mj[(g + (c >> 1) * 8) * MS + 8 * nt + 2 * t4 + (c & 1)] = sum3(lh[c], hl[c], hh[c]);
            }
            __syncwarp();
            {
                float lh[4] = {0.f, 0.f, 0.f, 0.f}, hl[4] = {0.f, 0.f, 0.f, 0.f}, hh[4] = {0.f, 0.f, 0.f, 0.f};
                mma3_tile(lh, hl, hh, 0, 2,
                          [&](int kb, int u) {
                              return TD[(16 * i + g + (u & 1) * 8) * MS + 16 * i + 8 * kb + t4 + (u >> 1) * 4];
                          },
                          [&](int kb, int u) { return Mj[(8 * kb + t4 + u * 4) * MS + 8 * nt + g]; });
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    TD[(16 * i + g + (c >> 1) * 8) * MS + 16 * j + 8 * nt + 2 * t4 + (c & 1)] =
                        -sum3(lh[c], hl[c], hh[c]);
            }
        }
        __syncthreads();
    }
    if constexpr (P::v_in_a(BF)) {
        // A is dead: the v rows go to its region.  Only the u0 half (warps
        // 0-3) reads them, so those 128 threads copy, wait and meet at a
        // named barrier while the w half starts.
        if (threadIdx.x < 128) {
            stage_v_rows<DV, C, BF>(vs, const_cast<unsigned char*>(b.vr), vrb, threadIdx.x, 128);
            cp_async_commit();
            cp_async_wait_all();
            asm volatile("bar.sync 1, 128;" ::: "memory");
        }
    }
    // [u0 | w] on the tensor cores: u0 = (T diag(beta)) V, w = (T diag(gamma)) K
    // with gamma_s = beta_s * D[s][0].  The first half of the warps takes the
    // u0 column blocks, the second half the w column blocks.  Row block r runs
    // over k blocks 0 .. 2r+1 (T is lower triangular); the scaled T fragment is
    // split once per k block and serves all the warp's column blocks.  For bf16
    // inputs k and v are exact in tf32: two products, (T_lo V) + (T_hi V);
    // otherwise three, ((T_lo V_hi) + (T_hi V_lo)) + (T_hi V_hi).
    {
        constexpr int D8 = DV / 8;  // column blocks per half (DK == DV)
        static_assert(DK == DV, "one column-block count for u0 and w");
        const int half = warp >= nwarps / 2, wi = warp - half * (nwarps / 2), nwh = nwarps / 2;
        constexpr int NJ = (D8 + 3) / 4;  // column blocks per warp with 8 warps
        const float* scale = half ? b.gam : b.bs;
        const unsigned char* src = half ? b.kr : b.vr;
        const int rb = half ? krb : vrb;
        // column 8 cb + g of a k row sits at 8 cb + pg once the rows are re-laid
        const int pg = (BF && half) ? 2 * (g & 3) + (g >> 2) : g;
        float* out = half ? wout : uout;
        const int ld = half ? ldw : ldu;
#pragma unroll 1
        for (int r = 0; r < NB; ++r) {
            float lh[NJ][4], hl[NJ][4], hh[NJ][4];
#pragma unroll
            for (int j = 0; j < NJ; ++j)
#pragma unroll
                for (int c = 0; c < 4; ++c) lh[j][c] = hl[j][c] = hh[j][c] = 0.f;
#pragma unroll 1
            for (int kb = 0; kb < 2 * r + 2; ++kb) {
                uint32_t ah[4], al[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int col = 8 * kb + t4 + (u >> 1) * 4;
                    tf32_split(fmul(TD[(16 * r + g + (u & 1) * 8) * MS + col], scale[col]), ah[u], al[u]);
                }
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    const int cb = wi + j * nwh;
                    if (cb < D8) {
                        uint32_t bh[2], bl[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const float x = ld_raw<BF>(src + (size_t)(8 * kb + t4 + 4 * u) * rb, 8 * cb + pg);
                            if constexpr (BF) bh[u] = __float_as_uint(x);
                            else tf32_split(x, bh[u], bl[u]);
                        }
                        mma_tf32(lh[j], al, bh);
                        if constexpr (!BF) mma_tf32(hl[j], ah, bl);
                        mma_tf32(hh[j], ah, bh);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                const int cb = wi + j * nwh;
                if (cb < D8) {
#pragma unroll
                    for (int hv = 0; hv < 2; ++hv) {
                        const int t = 16 * r + g + 8 * hv, col = 8 * cb + 2 * t4;
                        float x[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int c = 2 * hv + e;
                            x[e] = BF ? fadd(lh[j][c], hh[j][c]) : sum3(lh[j][c], hl[j][c], hh[j][c]);
                        }
                        *reinterpret_cast<float2*>(out + (int64_t)t * ld + col) = make_float2(x[0], x[1]);
                    }
                }
            }
        }
    }
    __syncthreads();
}

// Stage one chunk's raw k rows, v rows (unless PrepCfg::v_in_a) and gates
// (token rows tok0.., head h of [T, H, D] tensors, or of the decode buffers
// with H = 1) into the layout of prep_bufs, by cp.async; the caller commits,
// waits and synchronises.
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
    const int pvs = P::v_in_a(bf16) ? 0 : pv;  // v rows staged here unless chunk_prep stages them
    for (int e = threadIdx.x; e < C * (pk + pvs); e += blockDim.x) {
        const int t = e / (pk + pvs), pc = e % (pk + pvs);
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
__device__ __forceinline__ void chunk_prep_any(const PrepBufs& b, int bf16, const VSrc& vs, float* uout, int ldu,
                                               float* wout, int ldw, float* dCout)
{
    if (bf16) chunk_prep<DK, DV, C, true>(b, vs, uout, ldu, wout, ldw, dCout);
    else chunk_prep<DK, DV, C, false>(b, vs, uout, ldu, wout, ldw, dCout);
}

// P_chunk part 1 for every full chunk: one CTA per (full chunk, head).  BF:
// bf16 inputs (else fp32), fixed at compile time.
template <int DK, int DV, int C, bool BF>
__global__ void __launch_bounds__(256, PrepCfg<DK, DV, C>::ctas_per_sm(BF))
k_prep(const void* __restrict__ k, const void* __restrict__ v, const float* __restrict__ alpha,
       const float* __restrict__ beta, const int32_t* __restrict__ cu, const int32_t* __restrict__ fco,
       const int32_t* __restrict__ err, int N, int H,
       float* __restrict__ w_ws, float* __restrict__ u_ws, float* __restrict__ dC_ws)
{
    constexpr int in_bf16 = BF;
    if (__ldg(err)) return;
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
    chunk_prep<DK, DV, C, BF>(b, VSrc{v, tok0, H, h, C}, u_ws + (int64_t)task * C * DV, DV,
                              w_ws + (int64_t)task * C * DK, DK, dC_ws + (int64_t)task * (C + 4));
}

}  // namespace gdn
