// gdn_cpr.cu -- host side of the C ABI declared in include/gdn_cpr.h.
//
// Validates arguments on the host, carves the caller's workspace and enqueues
// the kernels of kernels.cuh on the caller's stream.  It allocates no device
// memory and never synchronises.  Its only global mutable state is the
// failure-detection test setting (gdn_test_fault_injection) and the
// per-device address cache of gdn_cpr_forward_noalloc (end of file).
#include "gdn_cpr.h"
#include "kernels.cuh"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <mutex>

namespace {

using gdn::ChunkCfg;

constexpr size_t kAlign = 256;

// Failure-detection test setting (gdn_test_fault_injection): 0 = off; 1 = the
// fused forward kernel withholds its boundary-state publications and bounds
// each wait for one by g_fault_wait clocks.
std::atomic<int32_t> g_fault_mode{0};
std::atomic<int64_t> g_fault_wait{gdn::kWaitLimit};

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported(int32_t dk, int32_t dv, int32_t C)
{
    const bool d_ok = dk == dv && (dk == 16 || dk == 32 || dk == 64 || dk == 128);
    const bool c_ok = C == 16 || C == 32 || C == 64;
    return d_ok && c_ok;
}

bool dtype_ok(gdn_dtype_t t) { return t == GDN_F32 || t == GDN_BF16; }

struct SeqTotals {
    int64_t tasks = 0, full = 0, states = 0, maxc = 0;  // maxc: most chunk tasks of one sequence
    uint64_t hash = 0;  // gdn::cu_entry_hash summed over the host copy
};

// Host copy of cu_seqlens -> totals; false if invalid.
bool seq_totals(const int32_t* cu, int32_t N, int64_t T_total, int32_t C, SeqTotals* out)
{
    if (cu == nullptr || N < 0 || C <= 0) return false;
    if (cu[0] != 0 || (int64_t)cu[N] != T_total) return false;
    SeqTotals t;
    for (int32_t n = 0; n < N; ++n) {
        const int64_t L = (int64_t)cu[n + 1] - cu[n];
        if (L < 0) return false;
        t.tasks += (L + C - 1) / C;
        t.full += L / C;
        t.states += L / C + 1;
        t.maxc = std::max<int64_t>(t.maxc, (L + C - 1) / C);
        t.hash += gdn::cu_entry_hash(n, cu[n]);
    }
    t.hash += gdn::cu_entry_hash(N, cu[N]);
    if (t.tasks > INT32_MAX || t.states > INT32_MAX) return false;
    *out = t;
    return true;
}

// Workspace layout: [err | cto | fco | so | order | cumc | progress | w | u0 | dC],
// each 256-byte aligned (order, cumc and progress serve the fused chain + P_tok
// kernel; tok_next shares the error word's 16 bytes).
struct Workspace {
    int32_t* err;
    int32_t* tok_next;
    int32_t* cto;
    int32_t* fco;
    int32_t* so;
    int32_t* order;
    int32_t* cumc;
    int32_t* progress;
    float* w;
    float* u;
    float* dC;
    size_t bytes;
};

Workspace carve(void* base, int64_t max_full, int32_t N, int32_t H, int32_t dk, int32_t dv, int32_t C)
{
    Workspace ws{};
    size_t off = 0;
    auto take = [&](size_t n) {
        const size_t o = off;
        off = align_up(off + n);
        return o;
    };
    const size_t o_err = take(16);
    const size_t o_cto = take(sizeof(int32_t) * (size_t)(N + 1));
    const size_t o_fco = take(sizeof(int32_t) * (size_t)(N + 1));
    const size_t o_so = take(sizeof(int32_t) * (size_t)(N + 1));
    const size_t o_ord = take(sizeof(int32_t) * (size_t)(N + 1));
    const size_t o_cumc = take(sizeof(int32_t) * (size_t)(max_full + 2));  // maxc <= ceil(T / C)
    const size_t o_prog = take(sizeof(int32_t) * (size_t)N * H);
    const size_t o_w = take(sizeof(float) * (size_t)max_full * H * C * dk);
    const size_t o_u = take(sizeof(float) * (size_t)max_full * H * C * dv);
    const size_t o_dc = take(sizeof(float) * (size_t)max_full * H * (C + 4));
    ws.bytes = off;
    char* b = static_cast<char*>(base);
    if (b != nullptr) {
        ws.err = reinterpret_cast<int32_t*>(b + o_err);
        ws.cto = reinterpret_cast<int32_t*>(b + o_cto);
        ws.fco = reinterpret_cast<int32_t*>(b + o_fco);
        ws.so = reinterpret_cast<int32_t*>(b + o_so);
        ws.tok_next = reinterpret_cast<int32_t*>(b + o_err + 4);
        ws.order = reinterpret_cast<int32_t*>(b + o_ord);
        ws.cumc = reinterpret_cast<int32_t*>(b + o_cumc);
        ws.progress = reinterpret_cast<int32_t*>(b + o_prog);
        ws.w = reinterpret_cast<float*>(b + o_w);
        ws.u = reinterpret_cast<float*>(b + o_u);
        ws.dC = reinterpret_cast<float*>(b + o_dc);
    }
    return ws;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (the library does not link libcuda itself).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// Tensor map of a [T, H, D] token tensor for TMA boxes of D x 1 x `box`
// tokens (one head, consecutive tokens).  The base is 16-byte aligned (checked
// by the callers), and every stride is a multiple of 16 bytes.
bool token_map(CUtensorMap* map, const void* base, int64_t T, int32_t H, int32_t D, int bf16, int box)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (enc == nullptr || base == nullptr || T <= 0) return false;
    const cuuint64_t esz = bf16 ? 2 : 4;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)D * esz, (cuuint64_t)H * D * esz};
    const cuuint32_t boxd[3] = {(cuuint32_t)D, 1u, (cuuint32_t)box};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
               const_cast<void*>(base), dims, strides, boxd, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename K>
cudaError_t set_smem(K* kernel, size_t bytes)
{
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

struct FwdArgs {
    const void *q, *k, *v;
    const float *alpha, *beta, *state_in;
    const int32_t* cu;
    int32_t N, H;
    int in_bf16, out_bf16;
    void* o;
    float* states;
    const gdn_cache_t* cache;
    SeqTotals tot;
    int64_t T_total;
    Workspace ws;
    cudaStream_t stream;
    void* const* events;  // optional: 6 events around the kernels
};

inline void mark(void* const* events, int i, cudaStream_t s)
{
    if (events != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s);
}

template <int D, int C>
gdn_status_t launch_forward(const FwdArgs& a)
{
    using Cf = ChunkCfg<D, D, C>;
    using TC = gdn::TokCfg<D, D, C>;
    cudaError_t e = cudaSuccess;
    // Few (sequence, head) pairs leave most SMs idle during the serial chain:
    // then the chain and P_tok run as one cooperative kernel (one CTA per SM),
    // the P_tok tasks filling the SMs the chains do not use.
    const int npairs = a.N * a.H;
    int dev = 0, sms = 0, per_sm = 0;
    constexpr size_t fsm = gdn::FusedSmem<D, D, C>::BYTES;
    bool fused = false;
    if constexpr (gdn::FusedSmem<D, D, C>::OK) {
        if (a.tot.tasks > 0 && cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
            npairs + 16 <= sms && set_smem(gdn::k_chain_tok<D, D, C>, fsm) == cudaSuccess &&
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gdn::k_chain_tok<D, D, C>, 256, fsm) ==
                cudaSuccess &&
            per_sm >= 1)
            fused = true;
    }
    mark(a.events, 0, a.stream);
    gdn::k_tables<<<1, 1024, 0, a.stream>>>(a.cu, a.N, C, a.T_total, a.tot.tasks, a.tot.full, a.tot.states,
                                             a.tot.hash, a.ws.cto, a.ws.fco, a.ws.so, a.ws.err,
                                             fused ? a.ws.order : nullptr, a.ws.cumc, (int)a.tot.maxc,
                                             a.ws.progress, a.ws.tok_next, npairs);
    if ((e = cudaGetLastError()) != cudaSuccess) return GDN_ERR_CUDA;
    mark(a.events, 1, a.stream);
    if (a.tot.full > 0) {
        const size_t sm = gdn::PrepCfg<D, D, C>::bytes(a.in_bf16);
        auto kern = a.in_bf16 ? gdn::k_prep<D, D, C, true> : gdn::k_prep<D, D, C, false>;
        if (set_smem(kern, sm) != cudaSuccess) return GDN_ERR_CUDA;
        kern<<<(unsigned)(a.tot.full * a.H), Cf::THREADS, sm, a.stream>>>(
            a.k, a.v, a.alpha, a.beta, a.cu, a.ws.fco, a.ws.err, a.N, a.H, a.ws.w, a.ws.u, a.ws.dC);
        if ((e = cudaGetLastError()) != cudaSuccess) return GDN_ERR_CUDA;
    }
    mark(a.events, 2, a.stream);
    // TMA descriptors of q, k, v for the intra-chunk kernels (boxes of SC tokens of one head)
    CUtensorMap tmq, tmk, tmv;
    if (a.tot.tasks > 0 &&
        (!token_map(&tmq, a.q, a.T_total, a.H, D, a.in_bf16, TC::SC) ||
         !token_map(&tmk, a.k, a.T_total, a.H, D, a.in_bf16, TC::SC) ||
         !token_map(&tmv, a.v, a.T_total, a.H, D, a.in_bf16, TC::SC)))
        return GDN_ERR_CUDA;
    float* cacheRs = a.cache ? a.cache->rscale : nullptr;
    if constexpr (gdn::FusedSmem<D, D, C>::OK) if (fused) {
        mark(a.events, 3, a.stream);  // the chain has no separate time: it runs inside the next kernel
        const void* k = a.k;
        const float *alpha = a.alpha, *beta = a.beta, *state_in = a.state_in;
        const int32_t *cu = a.cu, *fco = a.ws.fco, *so = a.ws.so, *order = a.ws.order, *cumc = a.ws.cumc;
        int32_t *err = a.ws.err, *progress = a.ws.progress, *tok_next = a.ws.tok_next;
        int N = a.N, H = a.H, in_bf16 = a.in_bf16, out_bf16 = a.out_bf16, maxc = (int)a.tot.maxc;
        const float *w = a.ws.w, *u = a.ws.u, *dC = a.ws.dC;
        float* states = a.states;
        void* o = a.o;
        float* cacheR = a.cache ? a.cache->R : nullptr;
        const int32_t mode = g_fault_mode.load();
        int withhold = mode == 1 ? 1 : 0;
        long long wait_limit = mode == 1 ? (long long)g_fault_wait.load() : gdn::kWaitLimit;
        void* args[] = {&tmq, &tmk, &tmv, &k, &alpha, &beta, &state_in, &cu, &fco, &so, &err, &N, &H, &in_bf16,
                        &out_bf16, &w, &u, &dC, &states, &o, &cacheR, &cacheRs, &progress, &tok_next, &order,
                        &cumc, &maxc, &withhold, &wait_limit};
        if (cudaLaunchCooperativeKernel((const void*)gdn::k_chain_tok<D, D, C>, dim3((unsigned)sms), dim3(256), args,
                                        fsm, a.stream) != cudaSuccess ||
            cudaGetLastError() != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    if (!fused && a.N > 0) {
        constexpr size_t sm = gdn::ChainSmem<D, D, C>::BYTES;
        if (set_smem(gdn::k_chain<D, D, C>, sm) != cudaSuccess) return GDN_ERR_CUDA;
        gdn::k_chain<D, D, C><<<(unsigned)((int64_t)a.N * a.H), gdn::TcCfg<D, D, C>::THREADS, sm, a.stream>>>(
            a.k, a.state_in, a.cu, a.ws.fco, a.ws.so, a.ws.err, a.N, a.H, a.in_bf16, a.ws.w, a.ws.u, a.ws.dC,
            a.states);
        if ((e = cudaGetLastError()) != cudaSuccess) return GDN_ERR_CUDA;
    }
    if (!fused) mark(a.events, 3, a.stream);
    if (!fused && a.tot.tasks > 0) {
        constexpr size_t sm = TC::SMEM;
        if (set_smem(gdn::k_tok<D, D, C>, sm) != cudaSuccess) return GDN_ERR_CUDA;
        gdn::k_tok<D, D, C><<<(unsigned)(a.tot.tasks * a.H), TC::THREADS, sm, a.stream>>>(
            tmq, tmk, tmv, a.alpha, a.beta, a.cu, a.ws.cto, a.ws.so, a.ws.err, a.N, a.H, a.in_bf16, a.out_bf16,
            a.states, a.o, a.cache ? a.cache->R : nullptr, cacheRs);
        if ((e = cudaGetLastError()) != cudaSuccess) return GDN_ERR_CUDA;
    }
    mark(a.events, 4, a.stream);
    if (a.cache != nullptr && a.N > 0) {
        const gdn_cache_t& c = *a.cache;
        gdn::k_cache_fill<D, D, C><<<(unsigned)((int64_t)a.N * a.H), 256, 0, a.stream>>>(
            a.k, a.v, a.alpha, a.beta, a.cu, a.ws.so, a.ws.err, a.N, a.H, a.in_bf16, a.states, c.S_b, c.R, c.rscale,
            c.kbuf,
            c.vbuf, c.abuf, c.bbuf, c.pos);
        if ((e = cudaGetLastError()) != cudaSuccess) return GDN_ERR_CUDA;
    }
    mark(a.events, 5, a.stream);
    (void)e;
    return GDN_OK;
}

struct DecArgs {
    const void *q, *k, *v;
    const float *alpha, *beta;
    const gdn_cache_t* cache;
    int32_t N, H;
    int in_bf16, out_bf16;
    void* o;
    cudaStream_t stream;
    void* const* events;  // optional: 3 events around the kernels
    int may_resync;       // 0: the caller guarantees that no buffer fills in this step
};

template <int D, int C>
gdn_status_t launch_decode(const DecArgs& a)
{
    using DC = gdn::DecCfg<D, D>;
    const gdn_cache_t& c = *a.cache;
    const int64_t NH = (int64_t)a.N * a.H;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return GDN_ERR_CUDA;
    int per_sm = 0;
    if (set_smem(gdn::k_dec_tok<D, D, C>, DC::SMEM) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gdn::k_dec_tok<D, D, C>, DC::THREADS, DC::SMEM) !=
            cudaSuccess ||
        per_sm <= 0)
        return GDN_ERR_CUDA;
    const unsigned tgrid = (unsigned)std::min<int64_t>(NH, (int64_t)sms * per_sm);
    mark(a.events, 0, a.stream);
    gdn::k_dec_tok<D, D, C><<<tgrid, DC::THREADS, DC::SMEM, a.stream>>>(
        a.q, a.k, a.v, a.alpha, a.beta, a.in_bf16, a.out_bf16, c.R, c.rscale, c.kbuf, c.vbuf, c.abuf, c.bbuf,
        c.pos, a.o,
        (int)NH, c.status);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    mark(a.events, 1, a.stream);
    if (!a.may_resync) {  // no pair reaches the end of its buffer: nothing to resync
        mark(a.events, 2, a.stream);
        return GDN_OK;
    }
    // persistent: one CTA per SM, and at most 1024 (sequence, head) pairs per CTA
    const int64_t min_grid = (NH + 1023) / 1024;
    const unsigned rgrid = (unsigned)std::max<int64_t>(std::min<int64_t>(NH, sms), min_grid);
    if constexpr (2 * C <= D) {  // the resync in two kernels: P_chunk part 1 per pair, then the chain step
        const size_t psm = gdn::PrepCfg<D, D, C>::bytes(a.in_bf16);
        auto rprep = a.in_bf16 ? gdn::k_dec_rprep<D, D, C, true> : gdn::k_dec_rprep<D, D, C, false>;
        if (set_smem(rprep, psm) != cudaSuccess) return GDN_ERR_CUDA;
        rprep<<<(unsigned)NH, 256, psm, a.stream>>>(
            (int)NH, (const void*)c.kbuf, (const void*)c.vbuf, (const float*)c.abuf,
            (const float*)c.bbuf, c.pos, c.R);
        if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
        constexpr size_t ssm = gdn::RstepSmem<D, D, C>::BYTES;
        if (set_smem(gdn::k_dec_rstep<D, D, C>, ssm) != cudaSuccess) return GDN_ERR_CUDA;
        gdn::k_dec_rstep<D, D, C><<<rgrid, 256, ssm, a.stream>>>((int)NH, a.in_bf16, c.S_b, c.R, c.rscale,
                                                                 (const void*)c.kbuf, (const float*)c.abuf, c.pos,
                                                                 c.status);
        if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
        mark(a.events, 2, a.stream);
        return GDN_OK;
    }
    constexpr size_t sm = gdn::ResyncSmem<D, D, C>::BYTES;
    if (set_smem(gdn::k_dec_resync<D, D, C>, sm) != cudaSuccess) return GDN_ERR_CUDA;
    // programmatic dependent launch: the resync grid is scheduled while the
    // per-token step finishes and waits on the device (griddepcontrol.wait)
    // for its results, which hides its launch latency on the many steps that
    // have nothing to resync
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(rgrid);
    cfg.blockDim = dim3(ChunkCfg<D, D, C>::THREADS);
    cfg.dynamicSmemBytes = sm;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, gdn::k_dec_resync<D, D, C>, (int)NH, a.in_bf16, c.S_b, c.R, c.rscale,
                           (const void*)c.kbuf, (const void*)c.vbuf, (const float*)c.abuf, (const float*)c.bbuf,
                           c.pos, c.status) != cudaSuccess ||
        cudaGetLastError() != cudaSuccess)
        return GDN_ERR_CUDA;
    mark(a.events, 2, a.stream);
    return GDN_OK;
}

// Backward workspace: the forward's tables (err, cto, fco, so, ...), then the
// boundary adjoints Y_c (one d_v x d_k state per chunk-state slot), the
// chunk-local operands of every (chunk, head) task (k_bprep -> k_bgrad) and
// the per-CTA scratch of k_bgrad (at most kBwdMaxCtas resident CTAs).
constexpr int64_t kBwdMaxCtas = 148 * 4;

struct BwdWorkspace {
    Workspace t;  // tables only
    float *ybuf, *prep, *scratch;
    size_t bytes;
};

BwdWorkspace carve_bwd(void* base, int64_t T, int32_t N, int32_t H, int32_t dk, int32_t dv, int32_t C)
{
    BwdWorkspace w{};
    (void)dk;
    const Workspace tables = carve(nullptr, 0, N, H, dk, dv, C);  // the tables part alone
    size_t off = tables.bytes;
    auto take = [&](size_t n) {
        const size_t o = off;
        off = align_up(off + n);
        return o;
    };
    const int64_t max_states = T / C + N;   // >= sum_n (floor(L_n / C) + 1)
    const int64_t ntasks = (T / C + N) * H;  // >= chunk tasks x heads
    const int64_t ctas = std::min<int64_t>(std::max<int64_t>(ntasks, 1), kBwdMaxCtas);
    const size_t o_y = take(sizeof(float) * (size_t)max_states * H * dv * dk);
    const size_t o_pw = take(sizeof(float) * (size_t)ntasks * (2 * C * dv + C * C + 8 * C));  // gdn::BgCfg::PW
    const size_t o_sc = take(sizeof(float) * (size_t)ctas * 4 * C * dv);  // gdn::BgCfg::SCR (d_k = d_v)
    w.bytes = off;
    char* b = static_cast<char*>(base);
    if (b != nullptr) {
        w.t = carve(base, 0, N, H, dk, dv, C);
        w.ybuf = reinterpret_cast<float*>(b + o_y);
        w.prep = reinterpret_cast<float*>(b + o_pw);
        w.scratch = reinterpret_cast<float*>(b + o_sc);
    }
    return w;
}

struct BwdArgs {
    const void *q, *k, *v, *dO;
    const float *alpha, *beta, *states, *dstate_out;
    const int32_t* cu;
    int32_t N, H;
    int in_bf16;
    float *dq, *dk, *dv, *dalpha, *dbeta, *dstate;
    SeqTotals tot;
    int64_t T_total;
    BwdWorkspace ws;
    cudaStream_t stream;
    void* const* events;  // optional: 4 events around the kernels
};

template <int D, int C>
gdn_status_t launch_backward(const BwdArgs& a)
{
    using BG = gdn::BgCfg<D, C>;
    using SC = gdn::ScanCfg<D, D, C>;
    mark(a.events, 0, a.stream);
    gdn::k_tables<<<1, 1024, 0, a.stream>>>(a.cu, a.N, C, a.T_total, a.tot.tasks, a.tot.full, a.tot.states,
                                             a.tot.hash, a.ws.t.cto, a.ws.t.fco, a.ws.t.so, a.ws.t.err, nullptr,
                                             nullptr, 0, nullptr, nullptr, 0);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    if (set_smem(gdn::k_bwd_scan<D, D, C>, SC::SMEM) != cudaSuccess) return GDN_ERR_CUDA;
    gdn::k_bwd_scan<D, D, C><<<(unsigned)((int64_t)a.N * a.H * SC::NT), SC::THREADS, SC::SMEM, a.stream>>>(
        a.q, a.k, a.alpha, a.beta, a.dO, a.cu, a.ws.t.so, a.ws.t.err, a.H, a.in_bf16, a.dstate_out, a.ws.ybuf,
        a.dstate);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    mark(a.events, 1, a.stream);
    const int64_t ntasks = a.tot.tasks * a.H;
    if (ntasks > 0) {
        const size_t psm = gdn::PrepCfg<D, D, C>::bytes(a.in_bf16);
        auto bprep = a.in_bf16 ? gdn::k_bprep<D, C, true> : gdn::k_bprep<D, C, false>;
        if (set_smem(bprep, psm) != cudaSuccess) return GDN_ERR_CUDA;
        bprep<<<(unsigned)ntasks, 256, psm, a.stream>>>(a.k, a.v, a.alpha, a.beta, a.cu, a.ws.t.cto, a.ws.t.err,
                                                        a.N, a.H, a.ws.prep);
        if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    }
    mark(a.events, 2, a.stream);
    if (ntasks > 0) {
        auto kern = a.in_bf16 ? gdn::k_bgrad<D, C, true> : gdn::k_bgrad<D, C, false>;
        if (set_smem(kern, BG::SMEM) != cudaSuccess) return GDN_ERR_CUDA;
        int dev = 0, sms = 0, occ = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, BG::THREADS, BG::SMEM) != cudaSuccess)
            return GDN_ERR_CUDA;
        // resident CTAs per SM: by shared memory and by tensor memory (512 columns per SM)
        const int per_sm = std::max(1, std::min<int>(occ, 512 / (int)BG::TMEM_COLS));
        const int64_t grid = std::min<int64_t>({ntasks, (int64_t)sms * per_sm, kBwdMaxCtas});
        kern<<<(unsigned)grid, BG::THREADS, BG::SMEM, a.stream>>>(
            a.q, a.k, a.v, a.alpha, a.beta, a.dO, a.states, a.ws.ybuf, a.dstate_out, a.cu, a.ws.t.cto, a.ws.t.so,
            a.ws.t.err, a.N, a.H, ntasks, a.ws.prep, a.dq, a.dk, a.dv, a.dalpha, a.dbeta, a.ws.scratch);
        if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    }
    mark(a.events, 3, a.stream);
    return GDN_OK;
}

#define GDN_DISPATCH(FN, D_, C_, ARGS)                              \
    switch (D_ * 1000 + C_) {                                       \
        case 16016: return FN<16, 16>(ARGS);                        \
        case 16032: return FN<16, 32>(ARGS);                        \
        case 16064: return FN<16, 64>(ARGS);                        \
        case 32016: return FN<32, 16>(ARGS);                        \
        case 32032: return FN<32, 32>(ARGS);                        \
        case 32064: return FN<32, 64>(ARGS);                        \
        case 64016: return FN<64, 16>(ARGS);                        \
        case 64032: return FN<64, 32>(ARGS);                        \
        case 64064: return FN<64, 64>(ARGS);                        \
        case 128016: return FN<128, 16>(ARGS);                      \
        case 128032: return FN<128, 32>(ARGS);                      \
        case 128064: return FN<128, 64>(ARGS);                      \
        default: return GDN_ERR_UNSUPPORTED;                        \
    }

}  // namespace

extern "C" {

const char* gdn_contract_id(void) { return "gdn-cpr-schedule-v6/NL8/ptok-scaled/prep-inverse-mma-tf32x3/chain-tcgen05-tf32x3-1acc"; }

const char* gdn_status_string(gdn_status_t s)
{
    switch (s) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case GDN_ERR_CUDA: return "CUDA launch failed";
        case GDN_ERR_WORKSPACE: return "workspace missing or too small";
        case GDN_ERR_TIMEOUT: return "a bounded device wait ran out (outputs incomplete)";
        case GDN_ERR_DEVICE_INPUT: return "device input disagrees with the host copy or is out of range";
    }
    return "unknown status";
}

gdn_status_t gdn_test_fault_injection(int32_t mode, int64_t wait_clocks)
{
    if (mode == 0) {
        g_fault_mode.store(0);
        g_fault_wait.store(gdn::kWaitLimit);
        return GDN_OK;
    }
    if (mode != 1 || wait_clocks < 1 || wait_clocks > gdn::kWaitLimit) return GDN_ERR_INVALID_ARG;
    g_fault_wait.store(wait_clocks);
    g_fault_mode.store(1);
    return GDN_OK;
}

int64_t gdn_num_chunk_states(const int32_t* cu_seqlens_host, int32_t num_seqs, int32_t C)
{
    if (cu_seqlens_host == nullptr || num_seqs < 0 || C <= 0) return -1;
    SeqTotals t;
    if (!seq_totals(cu_seqlens_host, num_seqs, cu_seqlens_host[num_seqs], C, &t)) return -1;
    return t.states;
}

size_t gdn_cpr_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t H, int32_t d_k, int32_t d_v,
                              int32_t C)
{
    if (total_tokens < 0 || num_seqs < 0 || H <= 0 || d_k <= 0 || d_v <= 0 || C <= 0) return 0;
    return carve(nullptr, total_tokens / C, num_seqs, H, d_k, d_v, C).bytes;
}

gdn_status_t gdn_cpr_forward_timed(const void* q, const void* k, const void* v, const float* alpha,
                                   const float* beta, const float* state_in, const int32_t* cu_seqlens,
                                   const int32_t* cu_seqlens_host, int32_t num_seqs, int64_t total_tokens,
                                   int32_t H, int32_t d_k, int32_t d_v, int32_t C, gdn_dtype_t in_dtype,
                                   gdn_dtype_t out_dtype, void* o, float* chunk_states,
                                   const gdn_cache_t* cache_out, void* workspace, size_t workspace_bytes,
                                   void* stream, void* const* events)
{
    if (num_seqs < 0 || total_tokens < 0 || H <= 0 || d_k <= 0 || d_v <= 0 || C <= 0)
        return GDN_ERR_INVALID_ARG;
    if (total_tokens > INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return GDN_ERR_INVALID_ARG;
    if (!supported(d_k, d_v, C)) return GDN_ERR_UNSUPPORTED;
    SeqTotals tot;
    if (!seq_totals(cu_seqlens_host, num_seqs, total_tokens, C, &tot)) return GDN_ERR_INVALID_ARG;
    if (cu_seqlens == nullptr || chunk_states == nullptr) return GDN_ERR_INVALID_ARG;
    if (!aligned16(chunk_states) || (state_in && !aligned16(state_in))) return GDN_ERR_INVALID_ARG;
    if (total_tokens > 0) {
        if (!q || !k || !v || !alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return GDN_ERR_INVALID_ARG;
    }
    if (cache_out != nullptr) {
        const gdn_cache_t& c = *cache_out;
        if (!c.S_b || !c.R || !c.rscale || !c.kbuf || !c.vbuf || !c.abuf || !c.bbuf || !c.pos)
            return GDN_ERR_INVALID_ARG;
        if (!aligned16(c.S_b) || !aligned16(c.R) || !aligned16(c.kbuf) || !aligned16(c.vbuf))
            return GDN_ERR_INVALID_ARG;
        if (total_tokens > 0 && (!k || !v || !alpha || !beta)) return GDN_ERR_INVALID_ARG;
    }
    const Workspace need = carve(nullptr, total_tokens / C, num_seqs, H, d_k, d_v, C);
    if (workspace == nullptr || workspace_bytes < need.bytes) return GDN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return GDN_ERR_INVALID_ARG;
    if ((int64_t)num_seqs * H > INT32_MAX || tot.tasks * H * 2 > INT32_MAX) return GDN_ERR_INVALID_ARG;

    FwdArgs a;
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.state_in = state_in;
    a.cu = cu_seqlens; a.N = num_seqs; a.H = H;
    a.in_bf16 = in_dtype == GDN_BF16; a.out_bf16 = out_dtype == GDN_BF16;
    a.o = o; a.states = chunk_states; a.cache = cache_out; a.tot = tot; a.T_total = total_tokens;
    a.ws = carve(workspace, total_tokens / C, num_seqs, H, d_k, d_v, C);
    a.stream = static_cast<cudaStream_t>(stream);
    a.events = events;
    if (num_seqs == 0) {  // no kernel runs: only the device status word is reset
        if (cudaMemsetAsync(a.ws.err, 0, sizeof(int32_t), a.stream) != cudaSuccess) return GDN_ERR_CUDA;
        for (int i = 0; i < 6; ++i) mark(events, i, a.stream);
        return GDN_OK;
    }
    GDN_DISPATCH(launch_forward, d_k, C, a)
}

gdn_status_t gdn_cpr_forward(const void* q, const void* k, const void* v, const float* alpha, const float* beta,
                             const float* state_in, const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                             int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k, int32_t d_v,
                             int32_t C, gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, void* o, float* chunk_states,
                             const gdn_cache_t* cache_out, void* workspace, size_t workspace_bytes, void* stream)
{
    return gdn_cpr_forward_timed(q, k, v, alpha, beta, state_in, cu_seqlens, cu_seqlens_host, num_seqs,
                                 total_tokens, H, d_k, d_v, C, in_dtype, out_dtype, o, chunk_states, cache_out,
                                 workspace, workspace_bytes, stream, nullptr);
}

size_t gdn_cpr_backward_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t H, int32_t d_k, int32_t d_v,
                                       int32_t C)
{
    if (total_tokens < 0 || num_seqs < 0 || H <= 0 || d_k <= 0 || d_v <= 0 || C <= 0) return 0;
    return carve_bwd(nullptr, total_tokens, num_seqs, H, d_k, d_v, C).bytes;
}

gdn_status_t gdn_cpr_backward_timed(const void* q, const void* k, const void* v, const float* alpha,
                                    const float* beta, const void* dO, const float* chunk_states,
                                    const float* dstate_out, const int32_t* cu_seqlens, const int32_t* cu_seqlens_host, int32_t num_seqs,
                                    int64_t total_tokens, int32_t H, int32_t d_k, int32_t d_v, int32_t C,
                                    gdn_dtype_t in_dtype, float* dq, float* dk, float* dv, float* dalpha,
                                    float* dbeta, float* dstate_in, void* workspace, size_t workspace_bytes,
                                    void* stream, void* const* events)
{
    if (num_seqs < 0 || total_tokens < 0 || total_tokens > INT32_MAX || H <= 0 || d_k <= 0 || d_v <= 0 || C <= 0)
        return GDN_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype)) return GDN_ERR_INVALID_ARG;
    if (!supported(d_k, d_v, C)) return GDN_ERR_UNSUPPORTED;
    SeqTotals tot;
    if (!seq_totals(cu_seqlens_host, num_seqs, total_tokens, C, &tot)) return GDN_ERR_INVALID_ARG;
    if (cu_seqlens == nullptr || chunk_states == nullptr || dstate_in == nullptr) return GDN_ERR_INVALID_ARG;
    if (!aligned16(chunk_states) || !aligned16(dstate_in) || (dstate_out && !aligned16(dstate_out)))
        return GDN_ERR_INVALID_ARG;
    if (total_tokens > 0) {
        if (!q || !k || !v || !alpha || !beta || !dO || !dq || !dk || !dv || !dalpha || !dbeta)
            return GDN_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dq) || !aligned16(dk) ||
            !aligned16(dv))
            return GDN_ERR_INVALID_ARG;
    }
    // grids of (sequence, head, row tile) and (chunk, head, row tile) index with 32-bit integers
    if ((int64_t)num_seqs * H * d_v > INT32_MAX || tot.tasks * H > INT32_MAX) return GDN_ERR_INVALID_ARG;
    const BwdWorkspace need = carve_bwd(nullptr, total_tokens, num_seqs, H, d_k, d_v, C);
    if (workspace == nullptr || workspace_bytes < need.bytes) return GDN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0) {  // no kernel runs: only the device status word is reset
        if (cudaMemsetAsync(workspace, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return GDN_ERR_CUDA;
        for (int i = 0; i < 4; ++i) mark(events, i, static_cast<cudaStream_t>(stream));
        return GDN_OK;
    }
    BwdArgs a;
    a.q = q; a.k = k; a.v = v; a.dO = dO; a.alpha = alpha; a.beta = beta; a.states = chunk_states;
    a.dstate_out = dstate_out;
    a.cu = cu_seqlens; a.N = num_seqs; a.H = H; a.in_bf16 = in_dtype == GDN_BF16;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dalpha = dalpha; a.dbeta = dbeta; a.dstate = dstate_in;
    a.tot = tot; a.T_total = total_tokens;
    a.ws = carve_bwd(workspace, total_tokens, num_seqs, H, d_k, d_v, C);
    a.stream = static_cast<cudaStream_t>(stream);
    a.events = events;
    GDN_DISPATCH(launch_backward, d_k, C, a)
}

gdn_status_t gdn_cpr_backward(const void* q, const void* k, const void* v, const float* alpha, const float* beta,
                              const void* dO, const float* chunk_states, const float* dstate_out,
                              const int32_t* cu_seqlens,
                              const int32_t* cu_seqlens_host, int32_t num_seqs, int64_t total_tokens, int32_t H,
                              int32_t d_k, int32_t d_v, int32_t C, gdn_dtype_t in_dtype, float* dq, float* dk,
                              float* dv, float* dalpha, float* dbeta, float* dstate_in, void* workspace,
                              size_t workspace_bytes, void* stream)
{
    return gdn_cpr_backward_timed(q, k, v, alpha, beta, dO, chunk_states, dstate_out, cu_seqlens, cu_seqlens_host,
                                  num_seqs, total_tokens, H, d_k, d_v, C, in_dtype, dq, dk, dv, dalpha, dbeta,
                                  dstate_in, workspace, workspace_bytes, stream, nullptr);
}

gdn_status_t gdn_decode_step_ex(const void* q, const void* k, const void* v, const float* alpha,
                                const float* beta, const gdn_cache_t* cache, int32_t num_seqs, int32_t H,
                                int32_t d_k, int32_t d_v, int32_t C, gdn_dtype_t in_dtype, gdn_dtype_t out_dtype,
                                void* o, int32_t may_resync, void* stream, void* const* events)
{
    if (num_seqs < 0 || H <= 0 || d_k <= 0 || d_v <= 0 || C <= 0) return GDN_ERR_INVALID_ARG;
    if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return GDN_ERR_INVALID_ARG;
    if (!supported(d_k, d_v, C)) return GDN_ERR_UNSUPPORTED;
    if ((int64_t)num_seqs * H > INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (cache == nullptr) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0) {
        for (int i = 0; i < 3; ++i) mark(events, i, static_cast<cudaStream_t>(stream));
        return GDN_OK;
    }
    const gdn_cache_t& c = *cache;
    if (!q || !k || !v || !alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
    if (!c.S_b || !c.R || !c.rscale || !c.kbuf || !c.vbuf || !c.abuf || !c.bbuf || !c.pos) return GDN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(c.S_b) || !aligned16(c.R) ||
        !aligned16(c.kbuf) || !aligned16(c.vbuf))
        return GDN_ERR_INVALID_ARG;
    DecArgs a;
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.cache = cache;
    a.N = num_seqs; a.H = H; a.in_bf16 = in_dtype == GDN_BF16; a.out_bf16 = out_dtype == GDN_BF16;
    a.o = o; a.stream = static_cast<cudaStream_t>(stream); a.events = events; a.may_resync = may_resync != 0;
    GDN_DISPATCH(launch_decode, d_k, C, a)
}

gdn_status_t gdn_decode_step_timed(const void* q, const void* k, const void* v, const float* alpha,
                                   const float* beta, const gdn_cache_t* cache, int32_t num_seqs, int32_t H,
                                   int32_t d_k, int32_t d_v, int32_t C, gdn_dtype_t in_dtype,
                                   gdn_dtype_t out_dtype, void* o, void* stream, void* const* events)
{
    return gdn_decode_step_ex(q, k, v, alpha, beta, cache, num_seqs, H, d_k, d_v, C, in_dtype, out_dtype, o, 1,
                              stream, events);
}

gdn_status_t gdn_decode_step(const void* q, const void* k, const void* v, const float* alpha, const float* beta,
                             const gdn_cache_t* cache, int32_t num_seqs, int32_t H, int32_t d_k, int32_t d_v,
                             int32_t C, gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, void* o, void* stream)
{
    return gdn_decode_step_timed(q, k, v, alpha, beta, cache, num_seqs, H, d_k, d_v, C, in_dtype, out_dtype, o,
                                 stream, nullptr);
}

}  // extern "C"

// ---------------------------------------------------------------- no-allocation forward
// Workspace for gdn_cpr_forward_noalloc: a fixed device array that lives in this
// library's module, so callers that cannot allocate device memory still get
// a CPR forward.  Every device that loads the library holds these bytes until
// the process exits.  All calls on a device share them.
namespace {

constexpr size_t kNoallocScratchBytes = (size_t)GDN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address must come
// from cudaGetSymbolAddress, called once per device with that device current.
gdn_status_t noalloc_scratch(void** out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return GDN_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return GDN_OK;
}

}  // namespace

// The device status word is the workspace's first 4 bytes (carve: err), for
// the forward and the backward alike.
extern "C" gdn_status_t gdn_read_device_status(const void* workspace, int32_t* status_out, void* stream)
{
    if (status_out == nullptr) return GDN_ERR_INVALID_ARG;
    const void* ws = workspace;
    if (ws == nullptr) {
        void* p = nullptr;
        const gdn_status_t st = noalloc_scratch(&p);
        if (st != GDN_OK) return st;
        ws = p;
    }
    if (cudaMemcpyAsync(status_out, ws, sizeof(int32_t), cudaMemcpyDefault, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return GDN_ERR_CUDA;
    return GDN_OK;
}

extern "C" gdn_status_t gdn_cpr_forward_noalloc(const void* q, const void* k, const void* v, const float* alpha,
                                                const float* beta, const float* state_in,
                                                const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                                                int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                                                int32_t d_v, int32_t C, gdn_dtype_t in_dtype,
                                                gdn_dtype_t out_dtype, void* o, float* chunk_states,
                                                const gdn_cache_t* cache_out, void* stream)
{
    if (num_seqs < 0 || total_tokens < 0 || H <= 0 || d_k <= 0 || d_v <= 0 || C <= 0)
        return GDN_ERR_INVALID_ARG;
    if (carve(nullptr, total_tokens / C, num_seqs, H, d_k, d_v, C).bytes > kNoallocScratchBytes)
        return GDN_ERR_WORKSPACE;  // the batch needs more than the fixed scratch holds
    void* ws = nullptr;
    const gdn_status_t st = noalloc_scratch(&ws);
    if (st != GDN_OK) return st;
    // Nothing in the workspace has to start at zero: every kernel writes its
    // part of it (offset tables, error word, w, u0, decays) before any read.
    return gdn_cpr_forward(q, k, v, alpha, beta, state_in, cu_seqlens, cu_seqlens_host, num_seqs, total_tokens,
                           H, d_k, d_v, C, in_dtype, out_dtype, o, chunk_states, cache_out, ws,
                           kNoallocScratchBytes, stream);
}
