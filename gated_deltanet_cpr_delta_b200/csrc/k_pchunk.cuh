// k_pchunk.cuh -- chunk-boundary update P_chunk part 2: k_chain, the fused chain + P_tok kernel,
// k_cache_fill (sm_100a).  Part 1 (the chunk-local precompute) is in k_prep.cuh.
#pragma once

#include "k_prep.cuh"
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
        tc_epilogue_S<DK, DV, C>(SR, th, d0, Klo);
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
    static constexpr size_t TOK = ((TokCfg<DK, DV, C>::SMEM + 127) / 128) * 128;  // one P_tok task, 128-byte aligned
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
k_chain_tok(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const void* __restrict__ k,
            const float* __restrict__ alpha, const float* __restrict__ beta, const float* __restrict__ state_in,
            const int32_t* __restrict__ cu, const int32_t* __restrict__ fco, const int32_t* __restrict__ so,
            int32_t* err, int N, int H, int in_bf16, int out_bf16, const float* __restrict__ w_ws,
            const float* __restrict__ u_ws, const float* __restrict__ dC_ws, float* states, void* __restrict__ o,
            float* __restrict__ cacheR, float* __restrict__ cacheRs, int32_t* progress, int32_t* tok_next,
            const int32_t* __restrict__ order, const int32_t* __restrict__ cumc, int maxc, int withhold,
            long long wait_limit)
{
    using Fs = FusedSmem<DK, DV, C>;
    static_assert(Fs::OK, "d_v = 128: two 128-thread P_tok tasks per CTA");
    volatile int32_t* verr = err;
    if (*verr) return;
    extern __shared__ __align__(128) float4 smem_a128[];  // TMA boxes need 128-byte alignment
    float* sm = reinterpret_cast<float*>(smem_a128);
    if ((int)blockIdx.x < N * H) {
        chain_run<DK, DV, C>(k, state_in, cu, fco, so, err, H, in_bf16, w_ws, u_ws, dC_ws, states, blockIdx.x,
                             progress, withhold, sm);
        __syncthreads();
    }
    const int half = threadIdx.x >> 7, tid = threadIdx.x & 127;
    float* tsm = sm + half * (Fs::TOK / 4);
    const HalfSync hs{2 + half};
    tok_context_init<DK, DV, C>(tsm, tid);
    hs();
    uint32_t phase = 0;
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
        if (!tok_task<DK, DV, C, true>(TokMaps{&tm_q, &tm_k, &tm_v}, alpha, beta, n, c, h, H, seq0,
                                       __ldg(cu + n + 1) - seq0, (int64_t)__ldg(so + n) + c, in_bf16, out_bf16,
                                       states, o, cacheR, cacheRs, tsm, tid, hs, phase, err))
            break;
    }
}

// Decode cache for a continuation: one CTA per (sequence, head).  The running
// state of a partial last chunk (R, rscale) comes from the intra-chunk kernel.
template <int DK, int DV, int C>
__global__ void __launch_bounds__(256)
k_cache_fill(const void* __restrict__ k, const void* __restrict__ v, const float* __restrict__ alpha,
             const float* __restrict__ beta, const int32_t* __restrict__ cu, const int32_t* __restrict__ so,
             const int32_t* __restrict__ err, int N, int H, int in_bf16, const float* __restrict__ states,
             float* S_b, float* R, float* rscale, void* kbuf, void* vbuf, float* abuf, float* bbuf, int32_t* pos)
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
    if (threadIdx.x == 0) {
        pos[nh] = p;
        if (p == 0) rscale[nh] = 1.0f;  // otherwise the intra-chunk kernel wrote the running scale
    }
}

}  // namespace gdn
