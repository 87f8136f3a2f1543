// schedule.cuh -- device primitives of the fp32 CPR arithmetic schedule.
//
// Every floating-point operation on the path goes through these helpers.
// Each is exactly one IEEE binary32 operation, rounded to nearest-even, with
// no flush-to-zero.  The compiler may not contract them into other operations.
// The fixed reduction tree over d_k follows the principle on the IsoExec summary
// page ("Achieving Parallelism Invariance": contiguous K leaves, FP32
// accumulation inside a leaf, a fixed binary tree over the leaves) and the
// commentary blog, section 8.  This project fixes NL = 8 leaves.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_cpr.h"

namespace gdn {

constexpr unsigned kFullMask = 0xffffffffu;
constexpr int kLeaves = 8;

__device__ __forceinline__ float fmul(float a, float b) { return __fmul_rn(a, b); }
__device__ __forceinline__ float fadd(float a, float b) { return __fadd_rn(a, b); }
__device__ __forceinline__ float fsub(float a, float b) { return __fsub_rn(a, b); }
__device__ __forceinline__ float ffma(float a, float b, float c) { return __fmaf_rn(a, b, c); }

// Two fp32 lanes in one 64-bit register, for the sm_100 packed instructions
// fma.rn.f32x2 / mul.rn.f32x2.  Each lane is rounded exactly like the scalar
// fma.rn.f32 / mul.rn.f32 (no flush-to-zero), so packing two independent
// chains changes no bit of either; it halves the issue slots they take.
typedef unsigned long long f2x;

__device__ __forceinline__ f2x pk2(float lo, float hi)
{
    f2x r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void up2(f2x x, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(x));
}

__device__ __forceinline__ f2x ffma2(f2x a, f2x b, f2x c)
{
    f2x d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ f2x fmul2(f2x a, f2x b)
{
    f2x d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// Partial results of the 8-leaf tree ((p0+p1)+(p2+p3)) + ((p4+p5)+(p6+p7)),
// pushed leaf by leaf (l = 0..7, known at compile time after unrolling).
// t0 holds the final value after leaf 7.
struct TreeAcc {
    float t0, t1, t2;
};

__device__ __forceinline__ void tree_push(TreeAcc& s, int l, float p)
{
    switch (l) {
        case 0: s.t0 = p; break;
        case 1: s.t0 = fadd(s.t0, p); break;
        case 2: s.t1 = p; break;
        case 3: s.t1 = fadd(s.t1, p); s.t0 = fadd(s.t0, s.t1); break;
        case 4: s.t1 = p; break;
        case 5: s.t1 = fadd(s.t1, p); break;
        case 6: s.t2 = p; break;
        default: s.t2 = fadd(s.t2, p); s.t1 = fadd(s.t1, s.t2); s.t0 = fadd(s.t0, s.t1); break;
    }
}

// tree(x, y) over DK elements held by one thread (x, y: any address space).
template <int DK>
__device__ __forceinline__ float tree_dot(const float* x, const float* y)
{
    constexpr int L = DK / kLeaves;
    TreeAcc s;
#pragma unroll
    for (int l = 0; l < kLeaves; ++l) {
        float acc = fmul(x[l * L], y[l * L]);
#pragma unroll
        for (int m = 1; m < L; ++m) acc = ffma(x[l * L + m], y[l * L + m], acc);
        tree_push(s, l, acc);
    }
    return s.t0;
}

// One leaf: x[0]*y[0], then ascending fused multiply-adds.
template <int L>
__device__ __forceinline__ float leaf_dot(const float* x, const float* y)
{
    float acc = fmul(x[0], y[0]);
#pragma unroll
    for (int m = 1; m < L; ++m) acc = ffma(x[m], y[m], acc);
    return acc;
}

// The tree when 4 consecutive lanes each hold two adjacent leaves (2p, 2p+1):
// every lane returns the same value, because fp32 addition is commutative bit
// for bit (lane 1 computes s1+s0, lane 0 computes s0+s1).
__device__ __forceinline__ float tree_4lanes(float leaf_a, float leaf_b)
{
    float s = fadd(leaf_a, leaf_b);                     // (p_{2p} + p_{2p+1})
    s = fadd(s, __shfl_xor_sync(kFullMask, s, 1));      // ((p0+p1)+(p2+p3)), ((p4+p5)+(p6+p7))
    s = fadd(s, __shfl_xor_sync(kFullMask, s, 2));      // full tree
    return s;
}

// ---------------------------------------------------------------- input/output
// 8 consecutive elements of a bf16 or fp32 tensor, widened exactly to fp32.
// `off` is an element offset; the address must be 16-byte aligned.
__device__ __forceinline__ void load8(const void* base, int64_t off, int bf16, float* o)
{
    if (bf16) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(base) + off));
        o[0] = __uint_as_float(u.x << 16); o[1] = __uint_as_float(u.x & 0xffff0000u);
        o[2] = __uint_as_float(u.y << 16); o[3] = __uint_as_float(u.y & 0xffff0000u);
        o[4] = __uint_as_float(u.z << 16); o[5] = __uint_as_float(u.z & 0xffff0000u);
        o[6] = __uint_as_float(u.w << 16); o[7] = __uint_as_float(u.w & 0xffff0000u);
    } else {
        const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + off);
        const float4 a = __ldg(p), b = __ldg(p + 1);
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
        o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return a | (b << 16);
}

// Store 8 consecutive fp32 values as bf16 (nearest-even) or fp32.
__device__ __forceinline__ void store8(void* base, int64_t off, int bf16, const float* x)
{
    if (bf16) {
        uint4 u;
        u.x = pack_bf16x2(x[0], x[1]); u.y = pack_bf16x2(x[2], x[3]);
        u.z = pack_bf16x2(x[4], x[5]); u.w = pack_bf16x2(x[6], x[7]);
        *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(base) + off) = u;
    } else {
        float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + off);
        p[0] = make_float4(x[0], x[1], x[2], x[3]);
        p[1] = make_float4(x[4], x[5], x[6], x[7]);
    }
}

__device__ __forceinline__ void store1(void* base, int64_t off, int bf16, float x)
{
    if (bf16) reinterpret_cast<__nv_bfloat16*>(base)[off] = __float2bfloat16_rn(x);
    else reinterpret_cast<float*>(base)[off] = x;
}

// Asynchronous global -> shared copies (cp.async; 16 bytes bypass L1, 4 bytes go through it).
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}

__device__ __forceinline__ void cp_async4(void* smem, const void* gmem)
{
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem));
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }
// Release store / bounded acquire wait on a global int (cross-CTA progress).
__device__ __forceinline__ void st_release_gpu(int32_t* p, int32_t v)
{
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int32_t ld_acquire_gpu(const int32_t* p)
{
    int32_t v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// The bound of every wait on another CTA's progress: 2^31 clocks, about a second.
constexpr long long kWaitLimit = 1ll << 31;

// Waits until *p >= v; false once `limit` clocks have passed.
__device__ __forceinline__ bool wait_at_least(const int32_t* p, int32_t v, long long limit)
{
    const long long t0 = clock64();
    while (ld_acquire_gpu(p) < v) {
        if (clock64() - t0 > limit) return false;
        __nanosleep(256);
    }
    return true;
}

// The device status word: keeps the first error recorded (a gdn_status_t).
__device__ __forceinline__ void record_error(int32_t* status, int32_t code)
{
    if (status != nullptr) atomicCAS(status, (int32_t)GDN_OK, code);
}

// All but the N most recently committed groups have landed.
template <int N>
__device__ __forceinline__ void cp_async_wait_n() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// All but the most recently committed group have landed.
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }


// ---------------------------------------------------------------- tensor-core tiles
// fp32 -> tf32 (round to nearest, ties away; low 13 bits zero) and the split
// x = hi + lo with hi = tf32(x), lo = tf32(x - hi).
__device__ __forceinline__ uint32_t tf32_of(float x)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void tf32_split(float x, uint32_t& hi, uint32_t& lo)
{
    hi = tf32_of(x);
    lo = tf32_of(__fsub_rn(x, __uint_as_float(hi)));
}

// d += a * b on one 16x8x8 tf32 tile (warp-wide, fp32 accumulate).  Fragment
// layouts (g = lane / 4, t = lane % 4):
//   a[0] = A[g][t], a[1] = A[g+8][t], a[2] = A[g][t+4], a[3] = A[g+8][t+4]
//   b[0] = B[t][g], b[1] = B[t+4][g]                      (B is K x N)
//   d[0] = D[g][2t], d[1] = D[g][2t+1], d[2] = D[g+8][2t], d[3] = D[g+8][2t+1]
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2])
{
    asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Largest n in [0, N) with tab[n] <= g (tab non-decreasing, tab[0] = 0 <= g < tab[N]).
__device__ __forceinline__ int find_seq(const int32_t* tab, int N, int g)
{
    int lo = 0, hi = N;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(tab + mid) <= g) lo = mid; else hi = mid;
    }
    return lo;
}

}  // namespace gdn
