// P_chunk part 2 (the boundary-state update) on the 5th-generation tensor
// cores: tcgen05.mma with fp32 accumulators in tensor memory (TMEM).
//
// One CTA owns one (sequence, head) state, all d_v <= 128 rows: the MMA tile
// is M = 128 rows (rows past d_v are zero).  Per chunk:
//   phase 1   E = S w^T            A = S   (TMEM, hi/lo split), B = w   (smem)
//   e_t[i]    = D[C][t] * (u0_t[i] - E[i][t])
//   phase 2   P = e k              A = e   (TMEM, hi/lo split), B = k^T (smem)
//   S'[i][j]  = D[C][0] * S[i][j] + P[i][j]
// Each fp32 operand x is split as hi = tf32_rna(x), lo = tf32_rna(x - hi).
// A phase accumulates its split products in ONE TMEM accumulator, in this
// order: lo*hi over the K blocks of 8 ascending, then hi*lo, then hi*hi.  k is
// exact in tf32 for bf16 inputs, so its lo product is absent there.  The
// epilogues then read one value per element.  The prefill chain and the decode
// resync call the same device functions, so both give the same bits.
//
// Thread roles (256 threads): thread 0 issues the MMAs; in the epilogues warp w
// reads TMEM lane quarter w % 4 (row i = 32 * (w % 4) + lane) and the half
// w / 4 of that row's columns.
#pragma once

#include "schedule.cuh"

namespace gdn {

// ------------------------------------------------------------- primitives
__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Warp-wide: allocate ncols TMEM columns; the base address lands in *slot.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Generic-proxy smem writes -> visible to the tensor core (async proxy).
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint64_t* mbar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(mbar)), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* mbar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P1;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, P1;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(mbar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity; gives up after ~2^31 clocks
// (about a second) and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* mbar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(mbar, parity))
        if (clock64() - t0 > (1ll << 31)) return false;
    return true;
}

// D[tmem] (+)= A[tmem] * B[smem desc]; kind::tf32, fp32 accumulate.
__device__ __forceinline__ void mma_tf32_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

// The mbarrier receives one arrive when all MMAs issued before it are complete.
__device__ __forceinline__ void mma_commit(uint64_t* mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(mbar))
                 : "memory");
}

// 8 consecutive TMEM columns of this thread's lane, then wait for the load.
__device__ __forceinline__ void tmem_ld8(uint32_t a0, float (&x)[8])
{
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "r"(a0)
        : "memory");
#pragma unroll
    for (int m = 0; m < 8; ++m) x[m] = __uint_as_float(r[m]);
}

__device__ __forceinline__ void tmem_st8(uint32_t a, const uint32_t (&v)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(a), "r"(v[0]),
                 "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, no swizzle.  Core matrices are 8
// rows x 16 bytes (128 contiguous bytes); lbo = byte step between the two
// 16-byte K halves of an 8-wide K block, sbo = byte step between 8-row groups.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// ------------------------------------------------------------- layout
template <int DK, int DV, int C>
struct TcCfg {
    static_assert(DK % 16 == 0 && DK <= 128 && DV <= 128 && C % 16 == 0 && C <= 64, "tile shapes");
    static constexpr int THREADS = 256;
    static constexpr uint32_t TMEM_COLS = 512;
    // TMEM columns.  Live ranges: S (phase 1 A) | D1 (phase 1 accumulator,
    // read by the e epilogue) | e (phase 2 A) | D2 (phase 2 accumulator, read
    // by the S' epilogue, which then writes S for the next chunk; D2 takes
    // S_hi's columns, which phase 1 no longer needs).
    static constexpr uint32_t S_HI = 0, S_LO = 128;
    static constexpr uint32_t D1 = 256;                  // C columns
    static constexpr uint32_t E_HI = 320, E_LO = 384;    // C columns each
    static constexpr uint32_t D2 = 0;                    // DK columns
    // smem operands (bytes): w [C rows][DK] and k^T [DK rows][C], K-major.
    static constexpr uint32_t LBO = 128;
    static constexpr uint32_t SBO_W = DK * 32;
    static constexpr uint32_t SBO_K = C * 32 + 16;   // 16-byte pad: the transposing stores hit distinct banks
    static constexpr int W_FLOATS = C * DK;
    static constexpr int K_FLOATS = (DK / 8) * (int)SBO_K / 4;
    // the k^T region [Klo | Khi] also stages the S' rows once phase 2 is done
    static constexpr int K_REGION = 2 * K_FLOATS > DV * DK ? 2 * K_FLOATS : DV * DK;
    // instruction descriptors: kind::tf32, fp32 accumulate, A and B K-major, M = 128
    static constexpr uint32_t idesc(int n)
    {
        return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    }
    static constexpr uint32_t IDESC1 = idesc(C), IDESC2 = idesc(DK);
    static_assert(E_LO + C <= TMEM_COLS && D2 + DK <= S_LO, "TMEM column map");
};

// ------------------------------------------------------------- staging
// w rows [C][DK] (row stride ldw floats, global or shared) -> hi/lo canonical
// B operands.  Eight consecutive threads store one 128-byte core-matrix column.
template <int DK, int DV, int C>
__device__ __forceinline__ void tc_stage_w(const float* src, int ldw, float* Whi, float* Wlo, int tid, int nthr)
{
    using T = TcCfg<DK, DV, C>;
    constexpr int ITEMS = C * DK / 4;
    for (int e = tid; e < ITEMS; e += nthr) {
        const int r8 = e & 7, c4 = (e >> 3) % (DK / 4), tg = (e >> 3) / (DK / 4);
        const float4 x = *reinterpret_cast<const float4*>(src + (int64_t)(tg * 8 + r8) * ldw + 4 * c4);
        uint32_t h[4], l[4];
        tf32_split(x.x, h[0], l[0]);
        tf32_split(x.y, h[1], l[1]);
        tf32_split(x.z, h[2], l[2]);
        tf32_split(x.w, h[3], l[3]);
        const int off = tg * (int)(T::SBO_W / 4) + c4 * (int)(T::LBO / 4) + r8 * 4;
        *reinterpret_cast<uint4*>(Whi + off) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(Wlo + off) = make_uint4(l[0], l[1], l[2], l[3]);
    }
}

// k of C tokens (rows of a [T, H, DK] input from token tok0, head h) -> k^T
// hi (and lo unless exact) canonical B operands [DK rows][C].
template <int DK, int DV, int C>
__device__ __forceinline__ void tc_stage_kT(const void* k, int64_t tok0, int H, int h, int bf16, float* Khi,
                                            float* Klo)
{
    using T = TcCfg<DK, DV, C>;
    constexpr int ITEMS = C * DK / 8;
    for (int e = threadIdx.x; e < ITEMS; e += blockDim.x) {
        const int tl = e & 3, jg = (e >> 2) % (DK / 8), blk = (e >> 2) / (DK / 8);
        float x[8];
        load8(k, ((tok0 + 4 * blk + tl) * H + h) * (int64_t)DK + 8 * jg, bf16, x);
        const int base = jg * (int)(T::SBO_K / 4) + blk * (int)(T::LBO / 4) + tl;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            if (bf16) {
                Khi[base + 4 * m] = x[m];  // a widened bf16 value is exact in tf32
            } else {
                uint32_t hi, lo;
                tf32_split(x[m], hi, lo);
                Khi[base + 4 * m] = __uint_as_float(hi);
                Klo[base + 4 * m] = __uint_as_float(lo);
            }
        }
    }
}

// ------------------------------------------------------------- the step
template <int DK>
struct TcThread {
    int q, hf, row;
    uint32_t lane_base;  // TMEM address of this warp's lane quarter, column 0
    __device__ TcThread(uint32_t tbase)
    {
        const int w = threadIdx.x >> 5;
        q = w & 3;
        hf = w >> 2;
        row = 32 * q + (threadIdx.x & 31);
        lane_base = tbase + ((uint32_t)(32 * q) << 16);
    }
};

// This thread's half row of S -> TMEM (hi, lo), then wait for the stores.
template <int DK, int DV, int C>
__device__ __forceinline__ void tc_put_state(const float (&SR)[DK / 2], const TcThread<DK>& th)
{
    using T = TcCfg<DK, DV, C>;
    const int j0 = th.hf * (DK / 2);
#pragma unroll
    for (int c8 = 0; c8 < DK / 16; ++c8) {
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) tf32_split(SR[8 * c8 + m], hi[m], lo[m]);
        tmem_st8(th.lane_base + T::S_HI + j0 + 8 * c8, hi);
        tmem_st8(th.lane_base + T::S_LO + j0 + 8 * c8, lo);
    }
    tmem_wait_st();
}

// Load this thread's half row of a state (rows [DV][DK] at src; zeros when
// src is null) into SR and TMEM; copy it to dst when non-null.
template <int DK, int DV, int C>
__device__ __forceinline__ void tc_load_state(float (&SR)[DK / 2], const TcThread<DK>& th, const float* src,
                                              float* dst)
{
    const int j0 = th.hf * (DK / 2);
#pragma unroll
    for (int j = 0; j < DK / 2; j += 4) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (src != nullptr && th.row < DV) x = *reinterpret_cast<const float4*>(src + (int64_t)th.row * DK + j0 + j);
        SR[j] = x.x; SR[j + 1] = x.y; SR[j + 2] = x.z; SR[j + 3] = x.w;
        if (dst != nullptr && th.row < DV) *reinterpret_cast<float4*>(dst + (int64_t)th.row * DK + j0 + j) = x;
    }
    tc_put_state<DK, DV, C>(SR, th);
}

// The pieces of one boundary update S <- P_chunk part 2 (S, chunk).  Before
// tc_issue_phase1 the chunk's w operands (Whi/Wlo, canonical) and S (TMEM) are
// in place and the CTA has passed fence.proxy.async + tcgen05 fence + barrier;
// before tc_issue_phase2 the same holds for k^T (Khi/Klo).  The issuing
// functions run on thread 0 only; the others run on every thread.

// Phase 1: E = S w^T, the three split products into one accumulator (Whi =
// Wlo + C * DK).
template <int DK, int DV, int C>
__device__ __forceinline__ void tc_issue_phase1(uint32_t tbase, const float* Wlo, uint64_t* mbar)
{
    using T = TcCfg<DK, DV, C>;
    tc_fence_after();
    const uint32_t wl = smem_u32(Wlo), wh = wl + 4u * T::W_FLOATS;
#pragma unroll 1
    for (int kb = 0; kb < DK / 8; ++kb)
        mma_tf32_ts(tbase + T::D1, tbase + T::S_LO + 8 * kb, smem_desc(wh + 256u * kb, T::LBO, T::SBO_W), T::IDESC1,
                    kb > 0);
#pragma unroll 1
    for (int kb = 0; kb < DK / 8; ++kb)
        mma_tf32_ts(tbase + T::D1, tbase + T::S_HI + 8 * kb, smem_desc(wl + 256u * kb, T::LBO, T::SBO_W), T::IDESC1,
                    1);
#pragma unroll 1
    for (int kb = 0; kb < DK / 8; ++kb)
        mma_tf32_ts(tbase + T::D1, tbase + T::S_HI + 8 * kb, smem_desc(wh + 256u * kb, T::LBO, T::SBO_W), T::IDESC1,
                    1);
    mma_commit(mbar);
}

// Phase 2: P = e k: e_lo k_hi, [e_hi k_lo,] e_hi k_hi into one accumulator
// (Khi = Klo + K_FLOATS; k_lo only when k is not exact in tf32).
template <int DK, int DV, int C>
__device__ __forceinline__ void tc_issue_phase2(uint32_t tbase, const float* Klo, int k_exact, uint64_t* mbar)
{
    using T = TcCfg<DK, DV, C>;
    tc_fence_after();
    const uint32_t kl = smem_u32(Klo), kh = kl + 4u * T::K_FLOATS;
#pragma unroll 1
    for (int kb = 0; kb < C / 8; ++kb)
        mma_tf32_ts(tbase + T::D2, tbase + T::E_LO + 8 * kb, smem_desc(kh + 256u * kb, T::LBO, T::SBO_K), T::IDESC2,
                    kb > 0);
    if (!k_exact) {
#pragma unroll 1
        for (int kb = 0; kb < C / 8; ++kb)
            mma_tf32_ts(tbase + T::D2, tbase + T::E_HI + 8 * kb, smem_desc(kl + 256u * kb, T::LBO, T::SBO_K),
                        T::IDESC2, 1);
    }
#pragma unroll 1
    for (int kb = 0; kb < C / 8; ++kb)
        mma_tf32_ts(tbase + T::D2, tbase + T::E_HI + 8 * kb, smem_desc(kh + 256u * kb, T::LBO, T::SBO_K), T::IDESC2,
                    1);
    mma_commit(mbar);
}

// Every thread: wait for the MMAs committed to mbar.  False (on every thread)
// if the wait timed out on any thread.
__device__ __forceinline__ bool tc_wait(uint64_t* mbar, uint32_t& parity)
{
    const bool ok = mbar_wait(mbar, parity);
    parity ^= 1u;
    if (__syncthreads_or(!ok)) return false;
    tc_fence_after();
    return true;
}

// e_t[i] = D[C][t] * (u0_t[i] - E[i][t]) (us[t * ldu + i] = u0_t[i],
// dCs[s] = D[C][s]) into TMEM as the phase-2 A operand.  Ends with a barrier,
// after which us and dCs may be overwritten; returns D[C][0].
template <int DK, int DV, int C>
__device__ __forceinline__ float tc_epilogue_e(const TcThread<DK>& th, const float* us, int ldu, const float* dCs)
{
    using T = TcCfg<DK, DV, C>;
    const int t0 = th.hf * (C / 2);
#pragma unroll
    for (int c8 = 0; c8 < C / 16; ++c8) {
        const uint32_t col = t0 + 8 * c8;
        float E[8];
        tmem_ld8(th.lane_base + T::D1 + col, E);
        uint32_t eh[8], el[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int t = t0 + 8 * c8 + m;
            const float e = th.row < DV ? fmul(dCs[t + 1], fsub(us[t * ldu + th.row], E[m])) : 0.f;
            tf32_split(e, eh[m], el[m]);
        }
        tmem_st8(th.lane_base + T::E_HI + t0 + 8 * c8, eh);
        tmem_st8(th.lane_base + T::E_LO + t0 + 8 * c8, el);
    }
    tmem_wait_st();
    const float d0 = dCs[0];
    tc_fence_before();
    __syncthreads();
    return d0;
}

// S' = d0 S + P on this thread's half row: into SR,
// TMEM (as the next chunk's phase-1 operand) and the rows [DV][DK] at `stage`
// (free smem; 16-byte chunks swizzled by row so that these row-per-thread
// writes are conflict-free).  Ends with a barrier.
template <int DK, int DV, int C>
__device__ __forceinline__ void tc_epilogue_S(float (&SR)[DK / 2], const TcThread<DK>& th, float d0, float* stage)
{
    using T = TcCfg<DK, DV, C>;
    constexpr int NC = DK / 4, SW = (NC < 8 ? NC : 8) - 1;
    const int j0 = th.hf * (DK / 2);
#pragma unroll
    for (int c8 = 0; c8 < DK / 16; ++c8) {
        float P[8];
        tmem_ld8(th.lane_base + T::D2 + j0 + 8 * c8, P);
#pragma unroll
        for (int m = 0; m < 8; ++m) SR[8 * c8 + m] = fadd(fmul(d0, SR[8 * c8 + m]), P[m]);
    }
    if (th.row < DV) {
#pragma unroll
        for (int j = 0; j < DK / 2; j += 4) {
            const int c = (j0 + j) / 4;
            *reinterpret_cast<float4*>(stage + th.row * DK + 4 * (c ^ (th.row & SW))) =
                make_float4(SR[j], SR[j + 1], SR[j + 2], SR[j + 3]);
        }
    }
    // every lane's accumulator reads are done before S (hi, lo) overwrites them
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tc_put_state<DK, DV, C>(SR, th);
    tc_fence_before();
    __syncthreads();
}

// The staged rows -> dst1 / dst2 (global rows [DV][DK], when non-null) with
// coalesced 16-byte stores, by threads tid = 0 .. nthr-1.
template <int DK, int DV>
__device__ __forceinline__ void tc_store_rows(const float* stage, float* dst1, float* dst2, int tid, int nthr)
{
    constexpr int NC = DK / 4, SW = (NC < 8 ? NC : 8) - 1;
    for (int f = tid; f < DV * NC; f += nthr) {
        const int r = f / NC, c = f % NC;
        const float4 x = *reinterpret_cast<const float4*>(stage + r * DK + 4 * (c ^ (r & SW)));
        if (dst1 != nullptr) *reinterpret_cast<float4*>(dst1 + (int64_t)r * DK + 4 * c) = x;
        if (dst2 != nullptr) *reinterpret_cast<float4*>(dst2 + (int64_t)r * DK + 4 * c) = x;
    }
}

// The whole update with every operand staged beforehand (the decode resync).
// Whi = Wlo + C * DK and Khi = Klo + K_FLOATS; the S' rows are staged in the
// k^T buffers once phase 2 is done with them.  Returns false if an MMA
// completion wait timed out (nothing more written).
template <int DK, int DV, int C>
__device__ __forceinline__ bool tc_step(float (&SR)[DK / 2], const TcThread<DK>& th, uint32_t tbase, uint64_t* mbar,
                                        uint32_t& parity, const float* Wlo, float* Klo, const float* us, int ldu,
                                        const float* dCs, int k_exact, float* dst1, float* dst2)
{
    if (threadIdx.x == 0) tc_issue_phase1<DK, DV, C>(tbase, Wlo, mbar);
    if (!tc_wait(mbar, parity)) return false;
    const float d0 = tc_epilogue_e<DK, DV, C>(th, us, ldu, dCs);
    if (threadIdx.x == 0) tc_issue_phase2<DK, DV, C>(tbase, Klo, k_exact, mbar);
    if (!tc_wait(mbar, parity)) return false;
    tc_epilogue_S<DK, DV, C>(SR, th, d0, Klo);
    tc_store_rows<DK, DV>(Klo, dst1, dst2, threadIdx.x, blockDim.x);
    __syncthreads();
    return true;
}

// k of C tokens held in registers between its global load and its store into
// the canonical k^T operands (so the load latency overlaps other work).  Item
// e covers token 4 * (e / (4 * (DK / 8))) + e % 4 and columns 8 * jg .. +7.
template <int DK, int DV, int C, int NT>
struct KPrefetch {
    static constexpr int ITEMS = C * DK / 8, NI = (ITEMS + NT - 1) / NT;
    uint4 raw[NI][2];
    __device__ __forceinline__ void load(const void* k, int64_t tok0, int H, int h, int bf16, int tid)
    {
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            const int e = tid + i * NT;
            if (e < ITEMS) {
                const int tl = e & 3, jg = (e >> 2) % (DK / 8), blk = (e >> 2) / (DK / 8);
                const int64_t off = ((tok0 + 4 * blk + tl) * H + h) * (int64_t)DK + 8 * jg;
                if (bf16) {
                    raw[i][0] = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(k) + off));
                } else {
                    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(k) + off);
                    raw[i][0] = __ldg(p);
                    raw[i][1] = __ldg(p + 1);
                }
            }
        }
    }
    __device__ __forceinline__ void store(float* Khi, float* Klo, int bf16, int tid) const
    {
        using T = TcCfg<DK, DV, C>;
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            const int e = tid + i * NT;
            if (e < ITEMS) {
                const int tl = e & 3, jg = (e >> 2) % (DK / 8), blk = (e >> 2) / (DK / 8);
                const int base = jg * (int)(T::SBO_K / 4) + blk * (int)(T::LBO / 4) + tl;
                const uint32_t w[8] = {raw[i][0].x, raw[i][0].y, raw[i][0].z, raw[i][0].w,
                                       raw[i][1].x, raw[i][1].y, raw[i][1].z, raw[i][1].w};
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    if (bf16) {
                        const uint32_t b = w[m >> 1];
                        Khi[base + 4 * m] = __uint_as_float((m & 1) ? (b & 0xffff0000u) : (b << 16));
                    } else {
                        uint32_t hi, lo;
                        tf32_split(__uint_as_float(w[m]), hi, lo);
                        Khi[base + 4 * m] = __uint_as_float(hi);
                        Klo[base + 4 * m] = __uint_as_float(lo);
                    }
                }
            }
        }
    }
};

}  // namespace gdn
