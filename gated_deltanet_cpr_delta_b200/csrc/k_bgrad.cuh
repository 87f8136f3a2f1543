// k_bgrad.cuh -- CPR backward: the per-chunk gradients as dense products on
// the 5th-generation tensor cores (sm_100a).
//
// The gradient of L = sum_t dO_t . o_t through one chunk of the gated delta
// rule (IsoExec summary page, section "Chunkwise-Parallel Recurrent (CPR)
// Gated DeltaNet"), written with chunk-sized matrices.  Tokens t, s, r are
// 0-indexed inside the chunk; D[t][s] = alpha_{s+1} ... alpha_t (D[t][t] = 1),
// g_t = D[t][0] (the decay from the chunk start through token t), gp_t =
// g_{t-1} (gp_0 = 1), dn_t = the decay from after token t to the chunk end.
// S0 is the forward's state at the chunk start, Y = dL/dS at its end, and
// T = (I + A)^-1 with A[t][s] = beta_t D[t][s] (k_t . k_s) (s < t), so that
//
//   Delta = u0 - w S0^T          (u0 = T diag(beta) V, w = T diag(beta g) K: P_chunk part 1)
//   U_t   = S_{t-1} k_t = gp_t S0 k_t + sum_{r<t} D[t-1][r] (k_r . k_t) Delta_r
//   Dd    = T^T (diag(dn) K Y^T + M dO),   M[s][u] = D[u][s] (k_s . q_u) (u >= s)
//   dv    = diag(beta) Dd,   dbeta_t = Dd_t . (v_t - alpha_t U_t)
//   dq    = diag(g) dO S0 + Xq K
//   dk    = diag(dn) Delta Y - diag(alpha beta gp) Dd S0 + X1 Q - X23 K
//   dalpha_t = psi_t - beta_t Dd_t . U_t
//
// with Xq[t][r] = D[t][r] (dO_t . Delta_r) (r <= t), X1[t][s] = D[s][t]
// (Delta_t . dO_s) (s >= t), X23[t][s] = D[s][t] beta_s (Delta_t . Dd_s) for
// s > t and alpha_t beta_t D[t-1][s] (Delta_s . Dd_t) for s < t, and psi_t =
// <dL/dS_t, S_{t-1}> expanded into S0, Y and pairwise token terms (below).
//
// Every product runs transposed, with the d-sized dimension (state rows i or
// key columns j) on the M = 128 rows of a tcgen05.mma.kind::tf32: A in tensor
// memory (one row per TMEM lane), B K-major in shared memory, fp32
// accumulators in tensor memory.  Products of two token-indexed matrices stack
// two of them on the M rows ([K; Q] K^T, [dO; Dd] Delta^T).  fp32 operands are
// split as hi = tf32_rna(x), lo = tf32_rna(x - hi) and a product is lo*hi +
// hi*lo + hi*hi in one accumulator; an operand exact in tf32 (bf16 inputs) has
// no lo product.  The backward has no bitwise contract; repeats give the same
// bits (no atomics; every sum has a fixed order).
//
// One CTA per SM walks the (chunk, head) tasks.  The chunk's tokens past its
// length (a sequence's last chunk) are padded with k = q = v = dO = 0,
// alpha = 1, beta = 0, which contribute nothing.  Intermediate token-by-feature
// matrices go through a per-CTA scratch in global memory (L2-resident).
#pragma once

#include "k_prep.cuh"
#include "k_tc.cuh"

namespace gdn {

template <int D, int C>
struct BgCfg {
    static_assert(D % 16 == 0 && D <= 128 && C % 16 == 0 && C <= 64, "tile shapes");
    static constexpr int THREADS = 512;
    static constexpr int BK = D > 2 * C ? D : 2 * C;  // widest K of a B operand
    static constexpr int ACOLS = 2 * BK;              // TMEM: A (hi | lo)
    static constexpr uint32_t S0C = ACOLS, S1C = ACOLS + C, S2C = ACOLS + 2 * C, S3C = ACOLS + 3 * C;  // accumulators
    static constexpr uint32_t TMEM_COLS = ACOLS + 4 * C <= 128 ? 128 : (ACOLS + 4 * C <= 256 ? 256 : 512);
    static_assert(ACOLS + 4 * C <= 512, "TMEM columns");
    static constexpr int LD = C + 1;  // row stride of the C x C matrices
    static constexpr int MAT = C * LD;
    // smem (floats): [B hi | B lo] [T, then DOD | N1, then DDD | M, then F | DM | KK, then E2b |
    // KQ, then E1 - E2b] vectors partials [bf16 token tiles q | k | dO]; each C x C buffer is
    // taken over by the second matrix once the first is dead
    static constexpr int B_OFF = 0;
    static constexpr int T_OFF = 2 * C * BK;
    static constexpr int N1_OFF = T_OFF + MAT;
    static constexpr int F_OFF = N1_OFF + MAT;
    static constexpr int DM_OFF = F_OFF + MAT;
    static constexpr int KK_OFF = DM_OFF + MAT;
    static constexpr int KQ_OFF = KK_OFF + MAT;
    static constexpr int VS = C + 4;
    enum { VA, VB, VG, VGP, VDN, VAV, VBV, VCV, VDB, VDU, NV };
    static constexpr int V_OFF = KQ_OFF + MAT;
    static constexpr int P_OFF = V_OFF + NV * VS;  // [4 quantities][4 lane quarters][C]
    static constexpr int YS_OFF = P_OFF + 16 * C;  // [16] warp partials of <Y, S0>
    static constexpr int TILE_OFF = (YS_OFF + 16 + 3) / 4 * 4;      // 16-byte aligned
    static constexpr int TILE_FL = 3 * C * D / 2;                   // three [C][D] bf16 tiles
    static constexpr int BAR_OFF = TILE_OFF + TILE_FL;
    static constexpr int FLOATS = BAR_OFF + 4;
    static constexpr size_t SMEM = sizeof(float) * (size_t)FLOATS;
    static constexpr int64_t SCR = 4 * (int64_t)C * D;  // per-CTA scratch floats: Delta | KS | dn KY | Dd
    // per-(chunk, head) operands written by k_bprep: u0 [C][D] | w [C][D] | T [C][C] | alpha, beta, g, gp, dn [C]
    static constexpr int64_t PW = 2 * (int64_t)C * D + C * C + 8 * C;
    static constexpr uint32_t idesc(int n)
    {
        return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    }
    static constexpr uint32_t IDESC = idesc(C);  // every product has N = C
};

// 4 consecutive elements (16-byte aligned for fp32, 8-byte for bf16) widened to fp32.
__device__ __forceinline__ float4 bg_load4(const void* base, int64_t off, int bf16)
{
    if (bf16) {
        const uint2 r = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(base) + off));
        return make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xffff0000u),
                           __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xffff0000u));
    }
    return __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + off));
}

__device__ __forceinline__ float bg_load1(const void* base, int64_t off, int bf16)
{
    return bf16 ? __uint_as_float((uint32_t)__ldg(reinterpret_cast<const uint16_t*>(base) + off) << 16)
                : __ldg(reinterpret_cast<const float*>(base) + off);
}

// 512 threads: warp w reads and writes TMEM lane quarter q = w % 4 (rows
// 32 q .. 32 q + 31, one per lane) and takes the 8-column groups g with
// g % 4 == p = w / 4.
constexpr int kBgThreads = 512, kBgParts = 4;

struct BgThread {
    int q, p, row;
    uint32_t lane_base;  // TMEM address of this warp's lane quarter, column 0
    __device__ explicit BgThread(uint32_t tbase)
    {
        const int w = threadIdx.x >> 5;
        q = w & 3;
        p = w >> 2;
        row = 32 * q + (threadIdx.x & 31);
        lane_base = tbase + ((uint32_t)(32 * q) << 16);
    }
};

// A operand rows in TMEM, K columns: this thread's lane row th.row and its
// column groups; f(m, k0, x) gives A[m][k0 .. k0+7].  hi goes to column
// chi + k, lo (when lo_too(g) for the group g = k0 / 8) to clo + k.  Every
// value is fetched before the first store (the stores are ordered with
// memory, so a load after one would wait for it).  Waits for its stores.
template <int K, typename L, typename F>
__device__ __forceinline__ void bg_put_a(const BgThread& th, uint32_t chi, uint32_t clo, L lo_too, F f)
{
    constexpr int NG = K / 8, GPT = (NG + kBgParts - 1) / kBgParts;
    float x[GPT][8];
#pragma unroll
    for (int j = 0; j < GPT; ++j) {
        const int g = th.p + kBgParts * j;
        if (g < NG) f(th.row, 8 * g, x[j]);
    }
#pragma unroll
    for (int j = 0; j < GPT; ++j) {
        const int g = th.p + kBgParts * j;
        if (g < NG) {
            uint32_t h[8], l[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) tf32_split(x[j][m], h[m], l[m]);
            tmem_st8(th.lane_base + chi + 8 * g, h);
            if (lo_too(g)) tmem_st8(th.lane_base + clo + 8 * g, l);
        }
    }
    tmem_wait_st();
}

// B operand [N rows][K] (K-major, no swizzle, 8-row groups K * 32 bytes apart)
// into hi (and lo, when non-null); f(r, c4) gives B[r][4 c4 .. 4 c4 + 3].
// Eight consecutive threads store one 128-byte core-matrix column; every
// value is fetched before the first store.
template <int N, int K, typename F>
__device__ __forceinline__ void bg_put_b(float* bh, float* bl, F f)
{
    constexpr int KQ4 = K / 4, TOT = N * KQ4, IT = (TOT + kBgThreads - 1) / kBgThreads;
    float4 x[IT];
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const int e = threadIdx.x + kBgThreads * it;
        if (e < TOT) x[it] = f(((e >> 3) / KQ4) * 8 + (e & 7), (e >> 3) % KQ4);
    }
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const int e = threadIdx.x + kBgThreads * it;
        if (e < TOT) {
            const int r8 = e & 7, c4 = (e >> 3) % KQ4, rg = (e >> 3) / KQ4;
            uint32_t h[4], l[4];
            tf32_split(x[it].x, h[0], l[0]);
            tf32_split(x[it].y, h[1], l[1]);
            tf32_split(x[it].z, h[2], l[2]);
            tf32_split(x[it].w, h[3], l[3]);
            const int off = rg * (K * 8) + c4 * 32 + r8 * 4;
            *reinterpret_cast<uint4*>(bh + off) = make_uint4(h[0], h[1], h[2], h[3]);
            if (bl != nullptr) *reinterpret_cast<uint4*>(bl + off) = make_uint4(l[0], l[1], l[2], l[3]);
        }
    }
}

// Thread 0: D[tmem d] (+)= A[tmem] B^T[smem] over the K blocks [kb0, kb1) of
// 8: lo*hi (unless A is exact), hi*lo (unless B is exact), hi*hi, in that
// order.  A block kb sits at columns a_hi + 8 kb / a_lo + 8 kb, B block kb at
// byte offset 256 kb (8-row groups sbo bytes apart).  acc: whether the first
// product adds to D.
__device__ __forceinline__ void bg_mma(uint32_t d, uint32_t a_hi, uint32_t a_lo, bool a_exact, const float* bh,
                                       const float* bl, bool b_exact, uint32_t sbo, int kb0, int kb1, uint32_t idesc,
                                       uint32_t& acc)
{
    const uint32_t h = smem_u32(bh), l = smem_u32(bl);
    if (!a_exact)
        for (int kb = kb0; kb < kb1; ++kb) {
            mma_tf32_ts(d, a_lo + 8 * kb, smem_desc(h + 256u * kb, 128u, sbo), idesc, acc);
            acc = 1;
        }
    if (!b_exact)
        for (int kb = kb0; kb < kb1; ++kb) {
            mma_tf32_ts(d, a_hi + 8 * kb, smem_desc(l + 256u * kb, 128u, sbo), idesc, acc);
            acc = 1;
        }
    for (int kb = kb0; kb < kb1; ++kb) {
        mma_tf32_ts(d, a_hi + 8 * kb, smem_desc(h + 256u * kb, 128u, sbo), idesc, acc);
        acc = 1;
    }
}

// Warp sum of 8 per-lane values: lane l ends with the sum of value l / 4
// (a fixed butterfly, so the order of the additions is fixed).
__device__ __forceinline__ float bg_warp_sum8(float (&x)[8])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const bool up = lane & 16;
        const float send = up ? x[j] : x[j + 4], keep = up ? x[j + 4] : x[j];
        x[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const bool up = lane & 8;
        const float send = up ? x[j] : x[j + 2], keep = up ? x[j + 2] : x[j];
        x[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    {
        const bool up = lane & 4;
        const float send = up ? x[0] : x[1], keep = up ? x[1] : x[0];
        x[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    x[0] += __shfl_xor_sync(0xffffffffu, x[0], 2);
    x[0] += __shfl_xor_sync(0xffffffffu, x[0], 1);
    return x[0];
}

// The chunk-local operands of every (chunk, head) task, chunks of C tokens
// padded as k_bgrad pads them: P_chunk part 1 (chunk_prep: u0, w and T) and
// the gates, into pw + task * BgCfg::PW.  One CTA per task; BF: bf16 inputs.
template <int D, int C, bool BF>
__global__ void __launch_bounds__(256, PrepCfg<D, D, C>::ctas_per_sm(BF))
k_bprep(const void* __restrict__ k, const void* __restrict__ v, const float* __restrict__ alpha,
        const float* __restrict__ beta, const int32_t* __restrict__ cu, const int32_t* __restrict__ cto,
        const int32_t* err, int N, int H, float* __restrict__ pw)
{
    constexpr int in_bf16 = BF;
    using P = PrepCfg<D, D, C>;
    if (*reinterpret_cast<volatile const int32_t*>(err)) return;
    extern __shared__ float4 smem_f4[];
    const int tid = threadIdx.x;
    const int64_t task = blockIdx.x;
    const int h = (int)(task % H);
    const int ct = (int)(task / H);
    const int n = find_seq(cto, N, ct);
    const int c = ct - __ldg(cto + n);
    const int seq0 = __ldg(cu + n);
    const int len = min(C, __ldg(cu + n + 1) - seq0 - c * C);
    const int64_t tok0 = (int64_t)seq0 + (int64_t)c * C;
    auto trow = [&](int t) { return (tok0 + t) * H + h; };
    const PrepBufs b = prep_bufs<D, D, C>(reinterpret_cast<unsigned char*>(smem_f4), in_bf16);
    const int esz = in_bf16 ? 2 : 4, pk = D * esz / 16;
    const int nparts = P::v_in_a(in_bf16) ? 1 : 2;  // k rows, and v rows unless chunk_prep stages them
    for (int e = tid; e < C * nparts * pk; e += blockDim.x) {
        const int t = e / (nparts * pk), pc = e % (nparts * pk), isv = pc >= pk, p = pc % pk;
        unsigned char* dst = const_cast<unsigned char*>(isv ? b.vr + (size_t)t * P::vrb(in_bf16)
                                                             : b.kr + (size_t)t * P::krb(in_bf16)) + 16 * p;
        if (t < len)
            cp_async16(dst, reinterpret_cast<const char*>(isv ? v : k) + trow(t) * D * esz + 16 * p);
        else
            *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    cp_async_commit();
    for (int t = tid; t < C; t += blockDim.x) {
        const_cast<float*>(b.as)[t] = t < len ? __ldg(alpha + trow(t)) : 1.0f;
        const_cast<float*>(b.bs)[t] = t < len ? __ldg(beta + trow(t)) : 0.0f;
    }
    cp_async_wait_all();
    __syncthreads();
    float* out = pw + task * BgCfg<D, C>::PW;
    chunk_prep<D, D, C, BF>(b, VSrc{v, tok0, H, h, len}, out, D, out + C * D, D, nullptr);
    float* oT = out + 2 * C * D;
    for (int e = tid; e < C * C; e += blockDim.x) {
        const int t = e / C, s = e % C;
        oT[e] = s <= t ? b.TD[t * P::MS + s] : 0.0f;  // T is lower triangular
    }
    float* ov = oT + C * C;
    for (int t = tid; t < C; t += blockDim.x) {
        ov[t] = b.as[t];
        ov[C + t] = b.bs[t];
        ov[2 * C + t] = b.d0[t];                         // g_t = D[t][0]
        ov[3 * C + t] = t == 0 ? 1.0f : b.d0[t - 1];     // gp_t
        ov[4 * C + t] = b.dC[t + 1];                     // dn_t
    }
}

// The per-chunk gradients of every (chunk, head) task; persistent.  BF16:
// the inputs are bf16 (else fp32), fixed at compile time so that no load
// carries a dtype branch.
template <int D, int C, bool BF16>
__global__ void __launch_bounds__(kBgThreads, 1)
k_bgrad(const void* __restrict__ q, const void* __restrict__ k, const void* __restrict__ v,
        const float* __restrict__ alpha, const float* __restrict__ beta, const void* __restrict__ dO,
        const float* __restrict__ states, const float* __restrict__ ybuf, const float* __restrict__ dstate_out,
        const int32_t* __restrict__ cu, const int32_t* __restrict__ cto, const int32_t* __restrict__ so,
        int32_t* err, int N, int H, int64_t ntasks, const float* __restrict__ pw,
        float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ dalpha,
        float* __restrict__ dbeta, float* __restrict__ scratch)
{
    using Cf = BgCfg<D, C>;
    constexpr int LD = Cf::LD, BK = Cf::BK, NG = C / 8;
    if (*reinterpret_cast<volatile const int32_t*>(err)) return;
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    float* Bh = sm + Cf::B_OFF;
    float* Bl = Bh + C * BK;
    float* Ts = sm + Cf::T_OFF;     // T
    float* DOD = Ts;                // then DOD[t][r] = dO_t . Delta_r
    float* N1 = sm + Cf::N1_OFF;    // N1 = T^T M
    float* DDD = N1;                // then DDD[t][r] = Dd_t . Delta_r
    float* FF = sm + Cf::F_OFF;     // M, later F
    float* DM = sm + Cf::DM_OFF;    // D[t][s]
    float* KK = sm + Cf::KK_OFF;    // k_t . k_s
    float* KQ = sm + Cf::KQ_OFF;    // k_t . q_s
    auto vec = [&](int which) { return sm + Cf::V_OFF + which * Cf::VS; };
    float *va = vec(Cf::VA), *vb = vec(Cf::VB), *vg = vec(Cf::VG), *vgp = vec(Cf::VGP), *vdn = vec(Cf::VDN);
    float *vav = vec(Cf::VAV), *vbv = vec(Cf::VBV), *vcv = vec(Cf::VCV), *vdb = vec(Cf::VDB), *vdu = vec(Cf::VDU);
    float* part = sm + Cf::P_OFF;
    float* ysp = sm + Cf::YS_OFF;
    uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + Cf::BAR_OFF);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Cf::BAR_OFF + 2);
    // bf16 inputs: the chunk's q, k, dO rows are staged once per task ([C][D] each)
    uint16_t* tq = reinterpret_cast<uint16_t*>(sm + Cf::TILE_OFF);
    uint16_t* tk = tq + C * D;
    uint16_t* tdo = tk + C * D;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (tid == 0) mbar_init(mbar, 1);
    if (tid < 32) tmem_alloc(tslot, Cf::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;
    const BgThread th(tbase);
    uint32_t parity = 0;
    float* gD = scratch + (int64_t)blockIdx.x * Cf::SCR;  // Delta [C][D]
    float* gKS = gD + C * D;                               // KS[t][i] = (S0 k_t)_i
    float* gKY = gKS + C * D;                              // dn_t (Y k_t)_i
    float* gDd = gKY + C * D;                              // Dd [C][D]
    const uint32_t a_hi = tbase, a_lo_D = tbase + D, a_lo_2C = tbase + 2 * C, a_lo_C = tbase + C;
    constexpr int in_bf16 = BF16 ? 1 : 0;
    constexpr bool ex = BF16;  // k, q, v, dO exact in tf32
    auto all_lo = [](int) { return true; };
    auto no_lo_if_exact = [&](int) { return !ex; };
    bool ok = true;

    // sync, issue (thread 0) and wait for the MMAs; false after a timeout
    auto run = [&](auto issue) -> bool {
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            issue();
            mma_commit(mbar);
        }
        return tc_wait(mbar, parity);
    };
    // per-column sums over the 128 lanes for the quantity slot qn: a warp
    // passes the 8 values of its column group g; after a barrier,
    // finish_sums gives out[t] = ((p0 + p1) + p2) + p3 over the lane quarters
    auto col_sum8 = [&](int qn, int g, float (&x)[8]) {
        const float s = bg_warp_sum8(x);
        if ((lane & 3) == 0) part[(qn * 4 + th.q) * C + 8 * g + (lane >> 2)] = s;
    };
    auto finish_sums = [&](int qn, float* out) {
        for (int t = tid; t < C; t += blockDim.x) {
            const float* pp = part + qn * 4 * C + t;
            out[t] = ((pp[0] + pp[C]) + pp[2 * C]) + pp[3 * C];
        }
    };

    for (int64_t task = blockIdx.x; task < ntasks && ok; task += gridDim.x) {
        const int h = (int)(task % H);
        const int ct = (int)(task / H);
        const int n = find_seq(cto, N, ct);
        const int c = ct - __ldg(cto + n);
        const int seq0 = __ldg(cu + n);
        const int Ln = __ldg(cu + n + 1) - seq0;
        const int64_t slot0 = __ldg(so + n);
        const int nchunks = (Ln + C - 1) / C;
        const int len = min(C, Ln - c * C);
        const int64_t tok0 = (int64_t)seq0 + (int64_t)c * C;
        const int64_t tb = (tok0 * H + h) * D;  // element offset of the chunk's first token row
        const int RS = H * D;                    // token row stride (elements)
        auto tok1 = [&](const void* base, int t, int i) { return bg_load1(base, tb + (t * RS + i), in_bf16); };
        // element (t, i), 4 elements (t, 4 c4 ..) and 8 elements (t, k0 ..) of q, k or dO (which = 0, 1, 2):
        // from the staged tiles for bf16 inputs, else from global memory
        auto tl1 = [&](int which, int t, int i) -> float {
            if constexpr (BF16) {
                return __uint_as_float((uint32_t)(which == 0 ? tq : which == 1 ? tk : tdo)[t * D + i] << 16);
            } else {
                return tok1(which == 0 ? q : which == 1 ? k : dO, t, i);
            }
        };
        auto tl4 = [&](int which, int t, int c4) -> float4 {
            if constexpr (BF16) {
                const uint2 r = *reinterpret_cast<const uint2*>((which == 0 ? tq : which == 1 ? tk : tdo) + t * D +
                                                                4 * c4);
                return make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xffff0000u),
                                   __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xffff0000u));
            } else {
                return bg_load4(which == 0 ? q : which == 1 ? k : dO, tb + (t * RS + 4 * c4), in_bf16);
            }
        };
        auto tl8 = [&](int which, int t, int k0, float (&x)[8]) {
            if constexpr (BF16) {
                const uint4 r = *reinterpret_cast<const uint4*>((which == 0 ? tq : which == 1 ? tk : tdo) + t * D + k0);
                const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    x[2 * m] = __uint_as_float(w[m] << 16);
                    x[2 * m + 1] = __uint_as_float(w[m] & 0xffff0000u);
                }
            } else {
                load8(which == 0 ? q : which == 1 ? k : dO, tb + (t * RS + k0), in_bf16, x);
            }
        };
        if constexpr (BF16) {  // stage the tiles (rows past the chunk's end are zero); waited for before KS
            constexpr int PR = D * 2 / 16;  // 16-byte pieces per row
            for (int e = tid; e < 3 * C * PR; e += blockDim.x) {
                const int which = e / (C * PR), rem = e % (C * PR), t = rem / PR, pc = rem % PR;
                uint16_t* dst = (which == 0 ? tq : which == 1 ? tk : tdo) + t * D + 8 * pc;
                if (t < len)
                    cp_async16(dst, reinterpret_cast<const uint16_t*>(which == 0 ? q : which == 1 ? k : dO) +
                                        tb + (int64_t)t * RS + 8 * pc);
                else
                    *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
            }
            cp_async_commit();
        }
        auto trow = [&](int t) { return (tok0 + t) * H + h; };  // row of [T, H] gates
        const float* S0 = states + ((slot0 + c) * H + h) * (int64_t)D * D;
        const float* Y = c + 1 < nchunks ? ybuf + ((slot0 + c + 1) * H + h) * (int64_t)D * D
                                         : (dstate_out != nullptr ? dstate_out + ((int64_t)n * H + h) * D * D
                                                                  : nullptr);

        // ---- chunk-local operands from k_bprep: u0, w, T and the gates
        const float* pwt = pw + task * Cf::PW;
        const float* gU = pwt;          // u0 [C][D]
        const float* gW = pwt + C * D;  // w [C][D]
        {
            const float* pT = pwt + 2 * C * D;
            const float* pv = pT + C * C;
            constexpr int TI = (C * C + kBgThreads - 1) / kBgThreads;
            float tv[TI];  // every value fetched before the first store
#pragma unroll
            for (int j = 0; j < TI; ++j) tv[j] = tid + j * kBgThreads < C * C ? pT[tid + j * kBgThreads] : 0.f;
#pragma unroll
            for (int j = 0; j < TI; ++j) {
                const int e = tid + j * kBgThreads;
                if (e < C * C) Ts[(e / C) * LD + e % C] = tv[j];
            }
            for (int t = tid; t < C; t += blockDim.x) {
                va[t] = pv[t];
                vb[t] = pv[C + t];
                vg[t] = pv[2 * C + t];
                vgp[t] = pv[3 * C + t];
                vdn[t] = pv[4 * C + t];
            }
            __syncthreads();
            for (int s = tid; s < C; s += blockDim.x) {  // DM[t][s] = D[t][s]: column s is a chain of products
                float d = 1.0f;
                for (int t = 0; t < s; ++t) DM[t * LD + s] = 0.0f;
                DM[s * LD + s] = d;
                for (int t = s + 1; t < C; ++t) {
                    d *= va[t];
                    DM[t * LD + s] = d;
                }
            }
        }

        // ---- E = S0 w^T (A = S0), then KS = S0 K^T (B = K)
        bg_put_a<D>(th, a_hi, a_lo_D, all_lo, [&](int m, int k0, float (&x)[8]) {
            if (m < D) {
                const float4 x0 = __ldg(reinterpret_cast<const float4*>(S0 + m * D + k0));
                const float4 x1 = __ldg(reinterpret_cast<const float4*>(S0 + m * D + k0 + 4));
                x[0] = x0.x; x[1] = x0.y; x[2] = x0.z; x[3] = x0.w;
                x[4] = x1.x; x[5] = x1.y; x[6] = x1.z; x[7] = x1.w;
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) x[j] = 0.f;
            }
        });
        bg_put_b<C, D>(Bh, Bl, [&](int r, int c4) { return *reinterpret_cast<const float4*>(gW + r * D + 4 * c4); });
        if constexpr (BF16) cp_async_wait_all();  // the tiles, visible to all after the barrier in run
        if (!(ok = run([&] {
                  uint32_t acc = 0;
                  bg_mma(tbase + Cf::S1C, a_hi, a_lo_D, false, Bh, Bl, false, D * 32, 0, D / 8, Cf::IDESC, acc);
              })))
            break;
        bg_put_b<C, D>(Bh, ex ? nullptr : Bl, [&](int r, int c4) {
            return r < len ? tl4(1, r, c4) : make_float4(0.f, 0.f, 0.f, 0.f);
        });
        if (!(ok = run([&] {
                  uint32_t acc = 0;
                  bg_mma(tbase + Cf::S2C, a_hi, a_lo_D, false, Bh, Bl, ex, D * 32, 0, D / 8, Cf::IDESC, acc);
              })))
            break;
        // ---- KY = Y K^T (A = Y; <Y, S0> on the way), then [K; Q] K^T (same B)
        {
            float ys = 0.f;
            bg_put_a<D>(th, a_hi, a_lo_D, all_lo, [&](int m, int k0, float (&x)[8]) {
#pragma unroll
                for (int j = 0; j < 8; ++j) x[j] = 0.f;
                if (m < D && Y != nullptr) {
                    const float4 y0 = __ldg(reinterpret_cast<const float4*>(Y + m * D + k0));
                    const float4 y1 = __ldg(reinterpret_cast<const float4*>(Y + m * D + k0 + 4));
                    const float4 s0 = __ldg(reinterpret_cast<const float4*>(S0 + m * D + k0));
                    const float4 s1 = __ldg(reinterpret_cast<const float4*>(S0 + m * D + k0 + 4));
                    x[0] = y0.x; x[1] = y0.y; x[2] = y0.z; x[3] = y0.w;
                    x[4] = y1.x; x[5] = y1.y; x[6] = y1.z; x[7] = y1.w;
                    ys += ((y0.x * s0.x + y0.y * s0.y) + (y0.z * s0.z + y0.w * s0.w)) +
                          ((y1.x * s1.x + y1.y * s1.y) + (y1.z * s1.z + y1.w * s1.w));
                }
            });
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) ys += __shfl_xor_sync(0xffffffffu, ys, o);
            if (lane == 0) ysp[warp] = ys;
        }
        if (!(ok = run([&] {
                  uint32_t acc = 0;
                  bg_mma(tbase + Cf::S3C, a_hi, a_lo_D, false, Bh, Bl, ex, D * 32, 0, D / 8, Cf::IDESC, acc);
              })))
            break;
        bg_put_a<D>(th, a_hi, a_lo_D, no_lo_if_exact, [&](int m, int k0, float (&x)[8]) {
            const int t = m % C;
            if (m < 2 * C && t < len) {
                tl8(m < C ? 1 : 0, t, k0, x);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) x[j] = 0.f;
            }
        });
        if (!(ok = run([&] {
                  uint32_t acc = 0;
                  bg_mma(tbase + Cf::S0C, a_hi, a_lo_D, ex, Bh, Bl, ex, D * 32, 0, D / 8, Cf::IDESC, acc);
              })))
            break;

        // ---- epilogue: KK, KQ; Delta, KS, dn KY to the scratch; cv_t = Delta_t . (Y k_t)
        float ysum = 0.f;
#pragma unroll
        for (int w = 0; w < kBgThreads / 32; ++w) ysum += ysp[w];
        {
            const int m = th.row, i = th.row;
            for (int g = th.p; g < NG; g += kBgParts) {
                const int t0 = 8 * g;
                float x[8], E[8], KS[8], KY[8], u0r[8];  // global values fetched first, all in flight
#pragma unroll
                for (int j = 0; j < 8; ++j) u0r[j] = i < D ? gU[(t0 + j) * D + i] : 0.f;
                tmem_ld8(th.lane_base + Cf::S0C + t0, x);
                tmem_ld8(th.lane_base + Cf::S1C + t0, E);
                tmem_ld8(th.lane_base + Cf::S2C + t0, KS);
                tmem_ld8(th.lane_base + Cf::S3C + t0, KY);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (m < C) KK[m * LD + t0 + j] = x[j];
                    else if (m < 2 * C) KQ[(t0 + j) * LD + m - C] = x[j];
                }
                float cv[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int t = t0 + j;
                    cv[j] = 0.f;
                    if (i < D) {
                        const float dl = u0r[j] - E[j];
                        gD[t * D + i] = dl;
                        gKS[t * D + i] = KS[j];
                        gKY[t * D + i] = vdn[t] * KY[j];
                        cv[j] = dl * KY[j];
                    }
                }
                col_sum8(0, g, cv);
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        finish_sums(0, vcv);
        // M[s][u] = D[u][s] KQ[s][u] (u >= s) into FF, then N1 = T^T M (upper
        // triangle), 2 x 4 outputs per thread, s over T's and M's nonzeros
        for (int e = tid; e < C * C; e += blockDim.x) {
            const int s_ = e / C, u = e % C;
            FF[s_ * LD + u] = u >= s_ ? DM[u * LD + s_] * KQ[s_ * LD + u] : 0.f;
        }
        __syncthreads();
        if (tid < C * C / 8) {
            const int t0 = 2 * (tid / (C / 4)), u0 = 4 * (tid % (C / 4));
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            const int s1 = min(C - 1, u0 + 3);
            for (int s_ = t0; s_ <= s1; ++s_) {
                const float a0 = Ts[s_ * LD + t0], a1 = Ts[s_ * LD + t0 + 1];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float bm = FF[s_ * LD + u0 + j];
                    acc[0][j] = fmaf(a0, bm, acc[0][j]);
                    acc[1][j] = fmaf(a1, bm, acc[1][j]);
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                N1[t0 * LD + u0 + j] = acc[0][j];
                N1[(t0 + 1) * LD + u0 + j] = acc[1][j];
            }
        }

        // ---- U^T = gp KS^T + Delta^T Xu^T, Xu[t][r] = D[t-1][r] KK[r][t] (r < t)
        bg_put_a<C>(th, a_hi, a_lo_C, all_lo, [&](int m, int k0, float (&x)[8]) {
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = m < D ? gD[(k0 + j) * D + m] : 0.f;
        });
        {  // accumulator S0C starts as gp_t KS[i][t]; every value fetched before the first store
            constexpr int GPT = (NG + kBgParts - 1) / kBgParts;
            float x[GPT][8];
#pragma unroll
            for (int jg = 0; jg < GPT; ++jg) {
                const int g = th.p + kBgParts * jg;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int t = 8 * g + j;
                    x[jg][j] = (g < NG && th.row < D) ? vgp[t] * gKS[t * D + th.row] : 0.f;
                }
            }
#pragma unroll
            for (int jg = 0; jg < GPT; ++jg) {
                const int g = th.p + kBgParts * jg;
                if (g < NG) {
                    uint32_t u[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) u[j] = __float_as_uint(x[jg][j]);
                    tmem_st8(th.lane_base + Cf::S0C + 8 * g, u);
                }
            }
            tmem_wait_st();
        }
        bg_put_b<C, C>(Bh, Bl, [&](int t, int c4) {
            float x[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = 4 * c4 + j;
                x[j] = r < t ? DM[(t - 1) * LD + r] * KK[r * LD + t] : 0.f;
            }
            return make_float4(x[0], x[1], x[2], x[3]);
        });
        if (!(ok = run([&] {
                  uint32_t acc = 1;
                  bg_mma(tbase + Cf::S0C, a_hi, a_lo_C, false, Bh, Bl, false, C * 32, 0, C / 8, Cf::IDESC, acc);
              })))
            break;

        // ---- Dd^T = [dn KY^T | dO^T] [T^T | N1]^T: K = 2C, A lo at column 2C
        bg_put_a<2 * C>(th, a_hi, a_lo_2C, [&](int g) { return g < C / 8 || !ex; },
                        [&](int m, int k0, float (&x)[8]) {
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int s_ = k0 + j;
                                x[j] = 0.f;
                                if (m < D) {
                                    if (s_ < C) x[j] = gKY[s_ * D + m];
                                    else if (s_ - C < len) x[j] = tl1(2, s_ - C, m);
                                }
                            }
                        });
        bg_put_b<C, 2 * C>(Bh, Bl, [&](int t, int c4) {
            float x[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int s_ = 4 * c4 + j;
                x[j] = s_ < C ? Ts[s_ * LD + t] : N1[t * LD + s_ - C];
            }
            return make_float4(x[0], x[1], x[2], x[3]);
        });
        if (!(ok = run([&] {
                  uint32_t acc = 0;
                  bg_mma(tbase + Cf::S1C, a_hi, a_lo_2C, false, Bh, Bl, false, 2 * C * 32, 0, C / 8, Cf::IDESC,
                         acc);
                  bg_mma(tbase + Cf::S1C, a_hi, a_lo_2C, ex, Bh, Bl, false, 2 * C * 32, C / 8, C / 4, Cf::IDESC,
                         acc);
              })))
            break;

        // ---- epilogue: dv, Dd to the scratch; sums for dbeta, Dd.U, bv
        {
            const int i = th.row;
            for (int g = th.p; g < NG; g += kBgParts) {
                const int t0 = 8 * g;
                float U[8], Dd[8], pdb[8], pdu[8], pbv[8], vr[8], ksr[8];  // global values fetched first
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int t = t0 + j;
                    vr[j] = (i < D && t < len) ? tok1(v, t, i) : 0.f;
                    ksr[j] = i < D ? gKS[t * D + i] : 0.f;
                }
                tmem_ld8(th.lane_base + Cf::S0C + t0, U);
                tmem_ld8(th.lane_base + Cf::S1C + t0, Dd);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int t = t0 + j;
                    pdb[j] = pdu[j] = pbv[j] = 0.f;
                    if (i < D) {
                        gDd[t * D + i] = Dd[j];
                        if (t < len) {
                            dv[tb + (t * RS + i)] = vb[t] * Dd[j];
                            pdb[j] = Dd[j] * (vr[j] - va[t] * U[j]);
                        }
                        pdu[j] = Dd[j] * U[j];
                        pbv[j] = Dd[j] * ksr[j];
                    }
                }
                col_sum8(1, g, pdb);
                col_sum8(2, g, pdu);
                col_sum8(3, g, pbv);
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        finish_sums(1, vdb);
        finish_sums(2, vdu);
        finish_sums(3, vbv);

        // ---- q1 = S0^T dO^T (A = S0^T), then av and the dq accumulator g q1
        bg_put_a<D>(th, a_hi, a_lo_D, all_lo, [&](int m, int k0, float (&x)[8]) {
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = m < D ? __ldg(S0 + (k0 + j) * D + m) : 0.f;
        });
        bg_put_b<C, D>(Bh, ex ? nullptr : Bl, [&](int r, int c4) {
            return r < len ? tl4(2, r, c4) : make_float4(0.f, 0.f, 0.f, 0.f);
        });
        if (!(ok = run([&] {
                  uint32_t acc = 0;
                  bg_mma(tbase + Cf::S2C, a_hi, a_lo_D, false, Bh, Bl, ex, D * 32, 0, D / 8, Cf::IDESC, acc);
              })))
            break;
        {
            const int j = th.row;
            for (int g = th.p; g < NG; g += kBgParts) {
                const int t0 = 8 * g;
                float q1[8], pav[8], qr[8];  // global values fetched first
                uint32_t sc[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) qr[e] = (j < D && t0 + e < len) ? tl1(0, t0 + e, j) : 0.f;
                tmem_ld8(th.lane_base + Cf::S2C + t0, q1);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    pav[e] = q1[e] * qr[e];
                    sc[e] = __float_as_uint(vg[t0 + e] * q1[e]);
                }
                tmem_st8(th.lane_base + Cf::S2C + t0, sc);
                col_sum8(0, g, pav);
            }
            tmem_wait_st();
        }
        // ---- dk accumulator: -(alpha beta gp) S0^T Dd^T (same A)
        bg_put_b<C, D>(Bh, Bl, [&](int t, int c4) {
            const float f = -(va[t] * vb[t]) * vgp[t];
            const float4 x = *reinterpret_cast<const float4*>(gDd + t * D + 4 * c4);
            return make_float4(f * x.x, f * x.y, f * x.z, f * x.w);
        });
        if (!(ok = run([&] {
                  uint32_t acc = 0;
                  bg_mma(tbase + Cf::S3C, a_hi, a_lo_D, false, Bh, Bl, false, D * 32, 0, D / 8, Cf::IDESC, acc);
              })))
            break;
        finish_sums(0, vav);

        // ---- dk += Y^T (dn Delta)^T (A = Y^T)
        bg_put_a<D>(th, a_hi, a_lo_D, all_lo, [&](int m, int k0, float (&x)[8]) {
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = (m < D && Y != nullptr) ? __ldg(Y + (k0 + j) * D + m) : 0.f;
        });
        bg_put_b<C, D>(Bh, Bl, [&](int t, int c4) {
            const float f = vdn[t];
            const float4 x = *reinterpret_cast<const float4*>(gD + t * D + 4 * c4);
            return make_float4(f * x.x, f * x.y, f * x.z, f * x.w);
        });
        if (!(ok = run([&] {
                  uint32_t acc = 1;
                  bg_mma(tbase + Cf::S3C, a_hi, a_lo_D, false, Bh, Bl, false, D * 32, 0, D / 8, Cf::IDESC, acc);
              })))
            break;

        // ---- [dO; Dd] Delta^T -> DOD, DDD
        bg_put_a<D>(th, a_hi, a_lo_D, all_lo, [&](int m, int k0, float (&x)[8]) {
            const int t = m % C;
            if (m < C && t < len) {
                tl8(2, t, k0, x);
            } else if (m >= C && m < 2 * C) {
                const float4 x0 = *reinterpret_cast<const float4*>(gDd + t * D + k0);
                const float4 x1 = *reinterpret_cast<const float4*>(gDd + t * D + k0 + 4);
                x[0] = x0.x; x[1] = x0.y; x[2] = x0.z; x[3] = x0.w;
                x[4] = x1.x; x[5] = x1.y; x[6] = x1.z; x[7] = x1.w;
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) x[j] = 0.f;
            }
        });
        bg_put_b<C, D>(Bh, Bl, [&](int t, int c4) { return *reinterpret_cast<const float4*>(gD + t * D + 4 * c4); });
        if (!(ok = run([&] {
                  uint32_t acc = 0;
                  bg_mma(tbase + Cf::S0C, a_hi, a_lo_D, false, Bh, Bl, false, D * 32, 0, D / 8, Cf::IDESC, acc);
              })))
            break;
        {
            const int m = th.row;
            for (int g = th.p; g < NG; g += kBgParts) {
                const int t0 = 8 * g;
                float x[8];
                tmem_ld8(th.lane_base + Cf::S0C + t0, x);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (m < C) DOD[m * LD + t0 + j] = x[j];
                    else if (m < 2 * C) DDD[(m - C) * LD + t0 + j] = x[j];
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- dalpha.  With E1[r][s] = DOD[s][r] KQ[r][s] and E2b[r][s] = beta_s DDD[s][r] KK[r][s]:
        //   F[r][t] = sum_{s>=t} E1[r][s] D[s][t] - sum_{s>t} E2b[r][s] D[s][t]
        //           = sum_{s>=t} (E1 - E2b)[r][s] D[s][t] + E2b[r][t]
        //   psi_t   = gp_t (dn_t <Y,S0> + sum_{s>=t} D[s][t] (av_s - beta_s bv_s) + beta_t bv_t)
        //           + sum_{r<t} D[t-1][r] (dn_t cv_r + F[r][t])
        float* Ed = KQ;  // E1 - E2b, in place over KQ (each element reads only its own KQ, KK)
        float* E2 = KK;  // E2b, in place over KK
        for (int e = tid; e < C * C; e += blockDim.x) {
            const int r = e / C, s_ = e % C;
            const float e2 = vb[s_] * DDD[s_ * LD + r] * KK[r * LD + s_];
            E2[r * LD + s_] = e2;
            Ed[r * LD + s_] = DOD[s_ * LD + r] * KQ[r * LD + s_] - e2;
        }
        __syncthreads();
        if (tid < C * C / 8) {  // F, 2 x 4 outputs per thread
            const int r0 = 2 * (tid / (C / 4)), t0 = 4 * (tid % (C / 4));
            float acc[2][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[0][j] = E2[r0 * LD + t0 + j];
                acc[1][j] = E2[(r0 + 1) * LD + t0 + j];
            }
            for (int s_ = t0; s_ < C; ++s_) {
                const float e0 = Ed[r0 * LD + s_], e1 = Ed[(r0 + 1) * LD + s_];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float dm = DM[s_ * LD + t0 + j];  // zero for s < t
                    acc[0][j] = fmaf(e0, dm, acc[0][j]);
                    acc[1][j] = fmaf(e1, dm, acc[1][j]);
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                FF[r0 * LD + t0 + j] = acc[0][j];
                FF[(r0 + 1) * LD + t0 + j] = acc[1][j];
            }
        }
        __syncthreads();
        {  // psi: 8 threads per token t, each over the s and r with s, r = sub (mod 8)
            const int t = tid >> 3, sub = tid & 7;
            float a = 0.f, b = 0.f;
            if (t < C) {
                for (int s_ = t + ((sub - t) & 7); s_ < C; s_ += 8)
                    a = fmaf(DM[s_ * LD + t], vav[s_] - vb[s_] * vbv[s_], a);
                for (int r = sub; r < t; r += 8) b = fmaf(DM[(t - 1) * LD + r], vdn[t] * vcv[r] + FF[r * LD + t], b);
            }
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                a += __shfl_xor_sync(0xffffffffu, a, o);
                b += __shfl_xor_sync(0xffffffffu, b, o);
            }
            if (t < len && sub == 0) {
                const float psi = vgp[t] * ((vdn[t] * ysum + a) + vb[t] * vbv[t]) + b;
                dalpha[trow(t)] = psi - vb[t] * vdu[t];
                dbeta[trow(t)] = vdb[t];
            }
        }

        // ---- dk += [Q^T | K^T] [X1 | -X23]^T; dq += K^T Xq^T  (A = [Q^T | K^T], K = 2C)
        bg_put_a<2 * C>(th, a_hi, a_lo_2C, no_lo_if_exact, [&](int m, int k0, float (&x)[8]) {
            const int which = k0 < C ? 0 : 1;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int s_ = (k0 + j) % C;
                x[j] = (m < D && s_ < len) ? tl1(which, s_, m) : 0.f;
            }
        });
        bg_put_b<C, 2 * C>(Bh, Bl, [&](int t, int c4) {
            float x[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int s_ = (4 * c4 + j) % C;
                if (4 * c4 < C) {  // X1[t][s] = D[s][t] DOD[s][t] (s >= t)
                    x[j] = s_ >= t ? DM[s_ * LD + t] * DOD[s_ * LD + t] : 0.f;
                } else {           // -X23[t][s]
                    float y = 0.f;
                    if (s_ > t) y = DM[s_ * LD + t] * vb[s_] * DDD[s_ * LD + t];
                    else if (s_ < t) y = va[t] * vb[t] * DM[(t - 1) * LD + s_] * DDD[t * LD + s_];
                    x[j] = -y;
                }
            }
            return make_float4(x[0], x[1], x[2], x[3]);
        });
        if (!(ok = run([&] {
                  uint32_t acc = 1;
                  bg_mma(tbase + Cf::S3C, a_hi, a_lo_2C, ex, Bh, Bl, false, 2 * C * 32, 0, C / 4, Cf::IDESC, acc);
              })))
            break;
        bg_put_b<C, C>(Bh, Bl, [&](int t, int c4) {  // Xq[t][r] = D[t][r] DOD[t][r] (r <= t)
            float x[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = 4 * c4 + j;
                x[j] = r <= t ? DM[t * LD + r] * DOD[t * LD + r] : 0.f;
            }
            return make_float4(x[0], x[1], x[2], x[3]);
        });
        // A = K^T: columns C.. of the hi part and 3C.. of the lo part; B block kb pairs with A block C/8 + kb
        if (!(ok = run([&] {
                  uint32_t acc = 1;
                  bg_mma(tbase + Cf::S2C, a_hi + C, a_lo_2C + C, ex, Bh, Bl, false, C * 32, 0, C / 8, Cf::IDESC,
                         acc);
              })))
            break;

        // ---- dq, dk
        {
            const int j = th.row;
            for (int g = th.p; g < NG; g += kBgParts) {
                const int t0 = 8 * g;
                float xq[8], xk[8];
                tmem_ld8(th.lane_base + Cf::S2C + t0, xq);
                tmem_ld8(th.lane_base + Cf::S3C + t0, xk);
                if (j < D) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int t = t0 + e;
                        if (t < len) {
                            dq[tb + (t * RS + j)] = xq[e];
                            dk[tb + (t * RS + j)] = xk[e];
                        }
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (!ok && tid == 0) record_error(err, GDN_ERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (tid < 32) {
        tc_fence_after();
        tmem_dealloc(tbase, Cf::TMEM_COLS);
    }
}

}  // namespace gdn
