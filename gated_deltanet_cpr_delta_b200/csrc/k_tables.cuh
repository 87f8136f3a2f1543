// k_tables.cuh -- offsets / validation kernel of the forward (sm_100a).
#pragma once

#include "schedule.cuh"

namespace gdn {

// ------------------------------------------------------------------ tables
// Position-sensitive hash of cu_seqlens: the wrapping sum over n of
// mix64((n << 32) | cu[n]) (the splitmix64 finalizer).  The host computes the
// same sum from its copy; the device recomputes it from the device copy.
__host__ __device__ inline uint64_t cu_entry_hash(int n, int32_t value)
{
    uint64_t z = ((uint64_t)(uint32_t)n << 32) | (uint64_t)(uint32_t)value;
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// One CTA.  For every sequence n (L_n = cu[n+1]-cu[n]):
//   cto[n] = sum_{m<n} ceil(L_m/C)      (chunk tasks of k_tok)
//   fco[n] = sum_{m<n} floor(L_m/C)     (full chunks: k_prep / k_chain)
//   so[n]  = sum_{m<n} (floor(L_m/C)+1) (chunk-state slots)
// and the totals at index N.  err[0], the call's device status word, becomes
// GDN_ERR_DEVICE_INPUT if the device cu_seqlens is invalid or disagrees with
// the host copy (totals or hash), else GDN_OK; every later kernel exits
// without writing while it is not GDN_OK.
// With order != NULL, also the tables of the fused chain + P_tok kernel
// (nt_n = ceil(L_n/C) chunk tasks of sequence n, maxc = max nt_n):
//   order[r]  sequences by nt_n descending (ties by n)
//   cumc[c]   = sum_n min(nt_n, c), c = 0..maxc (the chunk-major task offsets)
//   progress[0..npairs) = 0 and *tok_next = 0.
__global__ void k_tables(const int32_t* __restrict__ cu, int N, int C, int64_t T_total,
                         int64_t want_tasks, int64_t want_full, int64_t want_states, uint64_t want_hash,
                         int32_t* cto, int32_t* fco, int32_t* so, int32_t* err, int32_t* order, int32_t* cumc,
                         int maxc, int32_t* progress, int32_t* tok_next, int npairs)
{
    __shared__ long long wsum[3][32];
    __shared__ long long tot[3];
    __shared__ unsigned long long hsum;
    __shared__ int bad_any;
    const int tid = threadIdx.x, nth = blockDim.x;
    if (tid == 0) { bad_any = 0; hsum = 0ull; }
    __syncthreads();
    const int per = (N + nth - 1) / nth;
    const int n0 = min(N, tid * per), n1 = min(N, n0 + per);
    long long a = 0, b = 0, c = 0;
    unsigned long long hs = 0ull;
    int bad = 0;
    for (int n = n0; n < n1; ++n) {
        const int L = cu[n + 1] - cu[n];
        if (L < 0) bad = 1;
        const int Lc = L < 0 ? 0 : L;
        a += (Lc + C - 1) / C;
        b += Lc / C;
        c += Lc / C + 1;
        hs += cu_entry_hash(n, cu[n]);
    }
    if (tid == 0) hs += cu_entry_hash(N, cu[N]);
    atomicAdd(&hsum, hs);
    // block-wide exclusive scan of (a, b, c)
    const int lane = tid & 31, wid = tid >> 5;
    long long va = a, vb = b, vc = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const long long xa = __shfl_up_sync(kFullMask, va, d);
        const long long xb = __shfl_up_sync(kFullMask, vb, d);
        const long long xc = __shfl_up_sync(kFullMask, vc, d);
        if (lane >= d) { va += xa; vb += xb; vc += xc; }
    }
    if (lane == 31) { wsum[0][wid] = va; wsum[1][wid] = vb; wsum[2][wid] = vc; }
    __syncthreads();
    if (tid == 0) {
        long long ra = 0, rb = 0, rc = 0;
        for (int w = 0; w < (nth + 31) / 32; ++w) {
            const long long ta = wsum[0][w], tb = wsum[1][w], tc = wsum[2][w];
            wsum[0][w] = ra; wsum[1][w] = rb; wsum[2][w] = rc;
            ra += ta; rb += tb; rc += tc;
        }
        tot[0] = ra; tot[1] = rb; tot[2] = rc;
    }
    __syncthreads();
    long long ea = wsum[0][wid] + va - a, eb = wsum[1][wid] + vb - b, ec = wsum[2][wid] + vc - c;
    for (int n = n0; n < n1; ++n) {
        cto[n] = (int32_t)ea; fco[n] = (int32_t)eb; so[n] = (int32_t)ec;
        const int L = max(0, cu[n + 1] - cu[n]);
        ea += (L + C - 1) / C; eb += L / C; ec += L / C + 1;
    }
    if (bad) atomicOr(&bad_any, 1);
    __syncthreads();
    if (tid == 0) {
        cto[N] = (int32_t)tot[0]; fco[N] = (int32_t)tot[1]; so[N] = (int32_t)tot[2];
        const bool ok = !bad_any && cu[0] == 0 && (int64_t)cu[N] == T_total &&
                        tot[0] == want_tasks && tot[1] == want_full && tot[2] == want_states &&
                        hsum == want_hash;
        err[0] = ok ? (int32_t)GDN_OK : (int32_t)GDN_ERR_DEVICE_INPUT;
    }
    if (order != nullptr) {
        auto nt = [&](int m) { return (max(0, cu[m + 1] - cu[m]) + C - 1) / C; };
        for (int n = tid; n < N; n += nth) {
            const int a = nt(n);
            int rank = 0;
            for (int m = 0; m < N; ++m) {
                const int b = nt(m);
                rank += (b > a || (b == a && m < n)) ? 1 : 0;
            }
            order[rank] = n;
        }
        for (int c = tid; c <= maxc; c += nth) {
            int sum = 0;
            for (int m = 0; m < N; ++m) sum += min(nt(m), c);
            cumc[c] = sum;
        }
        for (int i = tid; i < npairs; i += nth) progress[i] = 0;
        if (tid == 0) *tok_next = 0;
    }
}

}  // namespace gdn
