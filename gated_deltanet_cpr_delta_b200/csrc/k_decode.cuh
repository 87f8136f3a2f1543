// k_decode.cuh -- decode step: k_dec_tok and k_dec_resync (sm_100a).
#pragma once

#include "k_ptok.cuh"
#include "k_pchunk.cuh"

namespace gdn {

// ------------------------------------------------------------------ decode
// One decode token per (sequence, head): P_tok on the running state
// rscale * R (the prefill's per-token step: tok_step_row), and the token
// appended to the buffer at slot pos.  Work item = (sequence-head, row tile).
// Persistent: CTA b takes the pairs b, b + grid, ..., each with all its row
// tiles in a row, so that once its last tile is done the CTA advances the
// pair's pos and rscale (every tile has read the old values by then).  A pair
// whose buffer is now full gets pos = C: k_dec_resync, which runs next, does
// its resync and sets pos = 0.  Each item's state rows and
// raw token stream into shared memory by cp.async, DecCfg::S - 1 items ahead
// of the one being computed, so several items' loads are in flight per CTA
// without holding registers.  Each lane's slice of a row (EPT contiguous
// floats) sits in its own padded slot, so the lane reads it conflict-free;
// the tile moves between global and shared memory a row per warp access
// (coalesced), in both directions.  Two stages and at most 128 registers a
// thread give 4 CTAs per SM (measured faster than 3 CTAs with three stages).
template <int DK, int DV>
struct DecCfg {
    using RS = RowSplit<DK>;
    static constexpr int RT = DV < 32 ? DV : 32;  // rows per item
    static constexpr int NT = DV / RT;
    static constexpr int THREADS = RT * RS::TPR;
    static constexpr int S = 2;                   // pipeline stages
    static constexpr int SLOT = RS::EPT + 4;      // floats per lane slice, padded
    static constexpr int RSTAGE = THREADS * SLOT; // state floats per stage
    static constexpr int RAWB = (2 * DK + RT) * 4 + 16;  // raw token bytes per stage (fp32 worst case) + gates, pos
    static constexpr int STAGE = RSTAGE + RAWB / 4;      // floats per stage
    static constexpr int TOKF = 2 * RS::KS + RT;         // widened token
    static constexpr size_t SMEM = sizeof(float) * ((size_t)S * STAGE + TOKF);
};

template <int DK, int DV, int C>
__global__ void __launch_bounds__(DecCfg<DK, DV>::THREADS, 4)
k_dec_tok(const void* __restrict__ q, const void* __restrict__ k, const void* __restrict__ v,
          const float* __restrict__ alpha, const float* __restrict__ beta, int in_bf16, int out_bf16,
          float* R, float* rscale, void* kbuf, void* vbuf, float* abuf, float* bbuf, int32_t* pos,
          void* __restrict__ o, int npairs, int32_t* status)
{
    using Cf = DecCfg<DK, DV>;
    using RS = typename Cf::RS;
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    float* ks = sm + Cf::S * Cf::STAGE;
    float* qs = ks + RS::KS;
    float* vs = qs + RS::KS;
    // the resync kernel that follows may be scheduled now; it waits for this
    // grid's completion before it reads anything
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int t = threadIdx.x;
    const int row = t / RS::TPR, part = t % RS::TPR;
    const int esz = in_bf16 ? 2 : 4;
    const int kp = DK * esz / 16, vp = Cf::RT * esz / 16;  // 16-byte pieces of k (= of q) and of the v rows
    const int el = 16 / esz;                               // elements per piece
    const int G = gridDim.x;
    auto rslot = [&](int st) { return sm + st * Cf::STAGE + t * Cf::SLOT; };
    // 16-byte chunk f of the tile (row-major) <-> its place in the lane slots
    constexpr int CPR = DK / 4, CPS = RS::EPT / 4;  // chunks per row, per lane slice
    auto chunk_slot = [&](int st, int f) {
        const int rr = f / CPR, c = f % CPR;
        return sm + st * Cf::STAGE + (rr * RS::TPR + c / CPS) * Cf::SLOT + 4 * (c % CPS);
    };
    auto raw = [&](int st) { return reinterpret_cast<unsigned char*>(sm + st * Cf::STAGE + Cf::RSTAGE); };

    // this CTA's j-th item: pair blockIdx.x + (j / NT) * grid, row tile j % NT
    auto item_pair = [&](int j) { return (int)blockIdx.x + (j / Cf::NT) * G; };
    auto fetch = [&](int j, int st) {  // item j -> stage st; always commits a group
        const int nh = item_pair(j), r = j % Cf::NT;
        if (nh < npairs) {
            const float* src = R + ((int64_t)nh * DV + r * Cf::RT) * DK;
            for (int f = t; f < Cf::RT * CPR; f += Cf::THREADS) cp_async16(chunk_slot(st, f), src + 4 * f);
            unsigned char* rw = raw(st);
            if (t < kp) cp_async16(rw + 16 * t, reinterpret_cast<const uint4*>(k) + (int64_t)nh * kp + t);
            else if (t < 2 * kp) cp_async16(rw + 16 * t, reinterpret_cast<const uint4*>(q) + (int64_t)nh * kp + (t - kp));
            else if (t < 2 * kp + vp)
                cp_async16(rw + 16 * t, reinterpret_cast<const uint4*>(v) + ((int64_t)nh * DV + r * Cf::RT) * esz / 16 +
                                            (t - 2 * kp));
            float* gates = reinterpret_cast<float*>(rw + 16 * (2 * kp + vp));
            if (t == 0) cp_async4(gates, alpha + nh);
            if (t == 1) cp_async4(gates + 1, beta + nh);
            if (t == 2) cp_async4(gates + 2, pos + nh);
            if (t == 3) cp_async4(gates + 3, rscale + nh);
        }
        cp_async_commit();
    };

#pragma unroll
    for (int j = 0; j < Cf::S - 1; ++j) fetch(j, j);
    for (int j = 0; item_pair(j) < npairs; ++j) {
        const int st = j % Cf::S;
        fetch(j + Cf::S - 1, (j + Cf::S - 1) % Cf::S);
        cp_async_wait_n<Cf::S - 1>();  // this item's copies (each thread's own) have landed
        __syncthreads();
        const int nh = item_pair(j), r = j % Cf::NT;
        const unsigned char* rw = raw(st);
        const float* gates = reinterpret_cast<const float*>(rw + 16 * (2 * kp + vp));
        const float a = gates[0], b = gates[1], cs = gates[3];
        const int p = __float_as_int(gates[2]);
        if (t < 2 * kp + vp) {  // widen the raw token
            const uint4 pc = *reinterpret_cast<const uint4*>(rw + 16 * t);
            const uint32_t w[4] = {pc.x, pc.y, pc.z, pc.w};
            float x[8];
            if (in_bf16) {
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    x[2 * m] = __uint_as_float(w[m] << 16);
                    x[2 * m + 1] = __uint_as_float(w[m] & 0xffff0000u);
                }
            } else {
#pragma unroll
                for (int m = 0; m < 4; ++m) x[m] = __uint_as_float(w[m]);
            }
            if (t < 2 * kp) {
                float* d = t < kp ? ks : qs;
                const int j0 = (t < kp ? t : t - kp) * el;
#pragma unroll
                for (int m = 0; m < 8; ++m)
                    if (m < el) d[RS::slot(j0 + m)] = x[m];
            } else {
                const int i0 = (t - 2 * kp) * el;
#pragma unroll
                for (int m = 0; m < 8; ++m)
                    if (m < el) vs[i0 + m] = x[m];
            }
            // append the raw token at slot p: k by tile 0, each tile its v rows
            if (p >= 0 && p < C) {
                if (t < kp && r == 0) reinterpret_cast<uint4*>(kbuf)[((int64_t)nh * C + p) * kp + t] = pc;
                if (t >= 2 * kp)
                    reinterpret_cast<uint4*>(vbuf)[(((int64_t)nh * C + p) * DV + r * Cf::RT) * esz / 16 +
                                                   (t - 2 * kp)] = pc;
            }
        }
        if (r == 0 && t == 0 && p >= 0 && p < C) {
            abuf[(int64_t)nh * C + p] = a;
            bbuf[(int64_t)nh * C + p] = b;
        }
        f2x Rp[RS::L];
        load_row_pairs<DK>(Rp, rslot(st));
        __syncthreads();  // the widened token is complete
        const bool valid = p >= 0 && p < C;  // an invalid position writes nothing
        if (!valid && t == 0) record_error(status, GDN_ERR_DEVICE_INPUT);
        if (valid) {
            const float cn = fmul(a, cs);
            const bool fold = !(cn >= kFoldTau);
            const float rc = fold ? 1.0f : __frcp_rn(cn);
            const float kq = tok_kq<DK>(ks + part * RS::PS, qs + part * RS::PS);
            const float ot = tok_step_row<DK>(Rp, ks + part * RS::PS, qs + part * RS::PS, vs[row], b, kq, cn, rc,
                                              fold);
            store_row_pairs<DK>(rslot(st), Rp);
            if (part == 0) store1(o, (int64_t)nh * DV + r * Cf::RT + row, out_bf16, ot);
        }
        __syncthreads();  // the new rows are in the slots
        if (valid) {
            float* dst = R + ((int64_t)nh * DV + r * Cf::RT) * DK;
            for (int f = t; f < Cf::RT * CPR; f += Cf::THREADS)
                *reinterpret_cast<float4*>(dst + 4 * f) = *reinterpret_cast<const float4*>(chunk_slot(st, f));
            if (r == Cf::NT - 1 && t == 0) {  // the pair's last tile: advance pos and the scale
                const float cn = fmul(a, cs);
                if (p + 1 < C) {
                    pos[nh] = p + 1;
                    rscale[nh] = cn >= kFoldTau ? cn : 1.0f;
                } else {
                    pos[nh] = C;  // full buffer: the resync follows
                }
            }
        }
        __syncthreads();  // ks / qs / vs and this stage are free again
    }
    cp_async_wait_all();
}

template <int DK, int DV, int C>
struct ResyncSmem {
    using P = PrepCfg<DK, DV, C>;
    using T = TcCfg<DK, DV, C>;
    static constexpr int WXS = DK + 4;                               // row stride of w
    static constexpr int WX_OFF = 0;                                 // [C][WXS] w, from chunk_prep
    static constexpr int US_OFF = WX_OFF + C * WXS;                  // [C][DV] u0
    static constexpr int DC_OFF = US_OFF + C * DV;                   // [C+4] D[C][.]
    // one region holds chunk_prep's raw rows and scratch, then (once w is
    // split) the canonical w lo | hi and k^T lo | hi operands (k^T's region
    // also stages S' after phase 2)
    static constexpr int R1_OFF = ((DC_OFF + C + 4 + 31) / 32) * 32;  // 128-byte aligned
    static constexpr int PREP_FL = (int)((P::bytes(0) + 3) / 4);
    static constexpr int TC_FL = 2 * T::W_FLOATS + T::K_REGION;
    static constexpr int R1_FL = PREP_FL > TC_FL ? PREP_FL : TC_FL;
    static constexpr int WLO_OFF = R1_OFF;
    static constexpr int KLO_OFF = R1_OFF + 2 * T::W_FLOATS;
    static constexpr int BAR_OFF = R1_OFF + ((R1_FL + 3) / 4) * 4;   // mbarrier (8 bytes) + TMEM base
    // at least 120 KB, so that one CTA fits per SM: each allocates all 512 TMEM columns
    static constexpr size_t USED = sizeof(float) * (BAR_OFF + 4);
    static constexpr size_t BYTES = USED > 120 * 1024 ? USED : 120 * 1024;
    static_assert(BYTES <= 232448, "fits the 227 KB of shared memory a CTA can have");
    static_assert(R1_OFF % 4 == 0 && US_OFF % 4 == 0 && KLO_OFF % 4 == 0 && BAR_OFF % 2 == 0, "alignment");
};

// Resyncs the pairs whose buffer k_dec_tok has just filled (pos == C):
// S_b <- P_chunk(S_b, buffer), R <- S_b, rscale <- 1, pos <- 0.  A step with
// no such pair costs one read of pos per pair.  P_chunk runs the same device functions as the prefill
// (chunk_prep, then the tcgen05 boundary step).  Persistent: CTA b handles
// (sequence, head) pairs b, b + grid, ...  Other positions are left as they
// are (k_dec_tok has advanced them, or recorded them as invalid).  If an MMA
// completion wait times
// out, the pairs this CTA had still to resync get pos = -1, are not written,
// and GDN_ERR_TIMEOUT goes to *status (when non-null).
template <int DK, int DV, int C>
__global__ void __launch_bounds__(256, 1)
k_dec_resync(int NH, int in_bf16, float* S_b, float* R, float* rscale, const void* kbuf, const void* vbuf,
             const float* abuf, const float* bbuf, int32_t* pos, int32_t* status)
{
    using Sm = ResyncSmem<DK, DV, C>;
    using T = TcCfg<DK, DV, C>;
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    float* wx = sm + Sm::WX_OFF;
    float* us = sm + Sm::US_OFF;
    float* dCs = sm + Sm::DC_OFF;
    unsigned char* r1 = reinterpret_cast<unsigned char*>(sm + Sm::R1_OFF);
    float* Wlo = sm + Sm::WLO_OFF;
    float* Whi = Wlo + T::W_FLOATS;
    float* Klo = sm + Sm::KLO_OFF;
    float* Khi = Klo + T::K_FLOATS;
    uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + Sm::BAR_OFF);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Sm::BAR_OFF + 2);

    // launched programmatically after k_dec_tok: wait for that grid's results
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // this CTA's pairs are blockIdx.x + i*gridDim.x: list the ones k_dec_tok
    // left at a full buffer (pos == C)
    __shared__ int todo[1024];
    __shared__ int ntodo;
    if (threadIdx.x == 0) ntodo = 0;
    __syncthreads();
    for (int nh = blockIdx.x + threadIdx.x * gridDim.x; nh < NH; nh += blockDim.x * gridDim.x) {
        if (pos[nh] == C) {
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
        prep_stage<DK, DV, C>(r1, kbuf, vbuf, abuf, bbuf, (int64_t)nh * C, 1, 0, in_bf16);
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
        chunk_prep_any<DK, DV, C>(prep_bufs<DK, DV, C>(r1, in_bf16), in_bf16, VSrc{vbuf, (int64_t)nh * C, 1, 0, C},
                                  us, DV, wx, Sm::WXS, dCs);
        tc_stage_w<DK, DV, C>(wx, Sm::WXS, Whi, Wlo, threadIdx.x, blockDim.x);
        tc_stage_kT<DK, DV, C>(kbuf, (int64_t)nh * C, 1, 0, in_bf16, Khi, Klo);
        float* Sg = S_b + (int64_t)nh * DV * DK;
        tc_load_state<DK, DV, C>(SR, th, Sg, nullptr);
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (!tc_step<DK, DV, C>(SR, th, tbase, mbar, parity, Wlo, Klo, us, DV, dCs, in_bf16, Sg,
                                R + (int64_t)nh * DV * DK))
            break;
        if (threadIdx.x == 0) {
            pos[nh] = 0;
            rscale[nh] = 1.0f;
        }
    }
    for (int r = it + threadIdx.x; r < nt; r += blockDim.x) pos[todo[r]] = -1;  // after a timeout
    if (it < nt && threadIdx.x == 0) record_error(status, GDN_ERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(tbase, T::TMEM_COLS);
    }
}


// The resync in two kernels, for 2C <= d (u0 and w of a chunk fit in one
// d x d state): on a step where buffers fill, the running state R of those
// pairs is dead until the resync rewrites it, so it holds their P_chunk
// part 1 operands in between.
//   k_dec_rprep: one CTA per pair, 3-4 CTAs per SM; a pair at pos == C runs
//     chunk_prep on its buffer: u0 -> R[0 .. C*d), w -> R[C*d .. 2*C*d).
//   k_dec_rstep: persistent, one CTA per SM; for each pair at pos == C the
//     tcgen05 step (tc_step) from S_b with w, k^T (from the buffer), u0
//     (staged from R into shared memory) and D[C][.] (from the buffered
//     gates, in chunk_prep's order of products), writing S_b and R; then
//     pos = 0, rscale = 1.
// The device functions and their operands are the single kernel's, so the
// results are bit for bit the same.
template <int DK, int DV, int C, bool BF>
__global__ void __launch_bounds__(256, PrepCfg<DK, DV, C>::ctas_per_sm(BF))
k_dec_rprep(int NH, const void* kbuf, const void* vbuf, const float* abuf, const float* bbuf,
            const int32_t* pos, float* R)
{
    constexpr int in_bf16 = BF;
    static_assert(2 * C * DV <= DV * DK && DK == DV, "u0 and w fit in one state");
    const int nh = blockIdx.x;
    if (nh >= NH || pos[nh] != C) return;
    extern __shared__ float4 smem_f4[];
    unsigned char* base = reinterpret_cast<unsigned char*>(smem_f4);
    // buffer rows are [nh][slot][D]: a [T, H=1, D] tensor starting at token nh*C
    prep_stage<DK, DV, C>(base, kbuf, vbuf, abuf, bbuf, (int64_t)nh * C, 1, 0, in_bf16);
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    float* out = R + (int64_t)nh * DV * DK;
    chunk_prep<DK, DV, C, BF>(prep_bufs<DK, DV, C>(base, in_bf16), VSrc{vbuf, (int64_t)nh * C, 1, 0, C}, out, DV,
                              out + C * DV, DK, nullptr);
}

template <int DK, int DV, int C>
struct RstepSmem {
    using T = TcCfg<DK, DV, C>;
    static constexpr int WLO_OFF = 0;
    static constexpr int KLO_OFF = WLO_OFF + 2 * T::W_FLOATS;
    static constexpr int DC_OFF = KLO_OFF + ((T::K_REGION + 3) / 4) * 4;  // [C + 4] D[C][.]
    static constexpr int AS_OFF = DC_OFF + ((C + 4 + 3) / 4) * 4;         // [C] the buffered alphas
    static constexpr int US_OFF = AS_OFF + ((C + 3) / 4) * 4;             // [C][DV] u0, from R
    static constexpr int WXS = DK + 4;                                     // row stride of w
    static constexpr int WX_OFF = US_OFF + C * DV;                         // [C][WXS] w, from R
    static constexpr int BAR_OFF = WX_OFF + C * WXS;
    // at least 120 KB, so that one CTA fits per SM: each allocates all 512 TMEM columns
    static constexpr size_t USED = sizeof(float) * (BAR_OFF + 4);
    static constexpr size_t BYTES = USED > 120 * 1024 ? USED : 120 * 1024;
    static_assert(BYTES <= 232448, "fits the 227 KB of shared memory a CTA can have");
};

template <int DK, int DV, int C>
__global__ void __launch_bounds__(256, 1)
k_dec_rstep(int NH, int in_bf16, float* S_b, float* R, float* rscale, const void* kbuf, const float* abuf,
            int32_t* pos, int32_t* status)
{
    using Sm = RstepSmem<DK, DV, C>;
    using T = TcCfg<DK, DV, C>;
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    float* Wlo = sm + Sm::WLO_OFF;
    float* Whi = Wlo + T::W_FLOATS;
    float* Klo = sm + Sm::KLO_OFF;
    float* Khi = Klo + T::K_FLOATS;
    float* dCs = sm + Sm::DC_OFF;
    float* as_ = sm + Sm::AS_OFF;
    float* us = sm + Sm::US_OFF;
    float* wx = sm + Sm::WX_OFF;
    uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + Sm::BAR_OFF);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Sm::BAR_OFF + 2);
    // this CTA's pairs are blockIdx.x + i*gridDim.x: list the ones at a full buffer
    __shared__ int todo[1024];
    __shared__ int ntodo;
    if (threadIdx.x == 0) ntodo = 0;
    __syncthreads();
    for (int nh = blockIdx.x + threadIdx.x * gridDim.x; nh < NH; nh += blockDim.x * gridDim.x) {
        if (pos[nh] == C) {
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
    // u0 rows [C][DV], then w rows [C][DK], parked in the pair's R by k_dec_rprep.  The
    // next pair's w and alphas are copied in while this pair's step runs, its u0 once
    // the step has consumed this one's.
    auto fetch_w = [&](int nh) {
        const float* Rn = R + (int64_t)nh * DV * DK;
        for (int f = threadIdx.x; f < C * DK / 4; f += blockDim.x) {
            const int t = f / (DK / 4), c4 = f % (DK / 4);
            cp_async16(wx + t * Sm::WXS + 4 * c4, Rn + C * DV + t * DK + 4 * c4);
        }
        for (int t = threadIdx.x; t < C; t += blockDim.x) cp_async4(as_ + t, abuf + (int64_t)nh * C + t);
        cp_async_commit();
    };
    auto fetch_u = [&](int nh) {
        const float* Rn = R + (int64_t)nh * DV * DK;
        for (int f = threadIdx.x; f < C * DV / 4; f += blockDim.x) cp_async16(us + 4 * f, Rn + 4 * f);
        cp_async_commit();
    };
    fetch_w(todo[0]);
    fetch_u(todo[0]);
    for (; it < nt; ++it) {
        const int nh = todo[it];
        float* Rn = R + (int64_t)nh * DV * DK;
        tc_stage_kT<DK, DV, C>(kbuf, (int64_t)nh * C, 1, 0, in_bf16, Khi, Klo);
        float* Sg = S_b + (int64_t)nh * DV * DK;
        cp_async_wait_all();
        __syncthreads();
        tc_stage_w<DK, DV, C>(wx, Sm::WXS, Whi, Wlo, threadIdx.x, blockDim.x);
        for (int s_ = threadIdx.x; s_ <= C; s_ += blockDim.x) {  // D[C][s], chunk_prep's order of products
            float d = 1.0f;
#pragma unroll
            for (int t = 0; t < C; ++t) {
                const float a = as_[t];
                if (t >= s_) d = fmul(d, a);
            }
            dCs[s_] = d;
        }
        tc_load_state<DK, DV, C>(SR, th, Sg, nullptr);
        fence_async_smem();
        tc_fence_before();
        __syncthreads();  // wx and as_ are consumed
        if (it + 1 < nt) fetch_w(todo[it + 1]);
        if (!tc_step<DK, DV, C>(SR, th, tbase, mbar, parity, Wlo, Klo, us, DV, dCs, in_bf16, Sg, Rn))
            break;
        if (threadIdx.x == 0) {
            pos[nh] = 0;
            rscale[nh] = 1.0f;
        }
        if (it + 1 < nt) fetch_u(todo[it + 1]);  // the step's epilogue has consumed us
    }
    cp_async_wait_all();
    for (int r = it + threadIdx.x; r < nt; r += blockDim.x) pos[todo[r]] = -1;  // after a timeout
    if (it < nt && threadIdx.x == 0) record_error(status, GDN_ERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(tbase, T::TMEM_COLS);
    }
}

}  // namespace gdn
