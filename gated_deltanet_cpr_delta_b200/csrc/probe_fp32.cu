// probe_fp32.cu -- measurement helper, not part of the layer's C ABI.
//
// Measures the sustained FP32 fused-multiply-add rate of the current GPU, the
// denominator of the FP32-bound roofline fractions the benchmark reports.
// Every thread runs 8 independent fma chains (scalar fma.rn.f32, or the packed
// fma.rn.f32x2 that the P_tok kernels use); 8 CTAs of 256 threads per SM keep
// enough warps in flight to hide the fma latency.  Built as its own library
// (libgdn_probe.so) so that the layer's library exports only the layer.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr int kChains = 8;
constexpr int kThreads = 256;
constexpr int kCtasPerSm = 8;

__global__ void __launch_bounds__(kThreads) k_probe_ffma(int iters, float b, float c, float* sink)
{
    float a[kChains];
#pragma unroll
    for (int i = 0; i < kChains; ++i) a[i] = (float)(threadIdx.x + i);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < kChains; ++i) asm volatile("fma.rn.f32 %0, %0, %1, %2;" : "+f"(a[i]) : "f"(b), "f"(c));
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kChains; ++i) s += a[i];
    if (s == 1234.5f) sink[blockIdx.x] = s;  // never true for the inputs used; keeps the chains alive
}

__global__ void __launch_bounds__(kThreads) k_probe_ffma2(int iters, float b, float c, float* sink)
{
    unsigned long long a[kChains], bb, cc;
    asm("mov.b64 %0, {%1, %1};" : "=l"(bb) : "f"(b));
    asm("mov.b64 %0, {%1, %1};" : "=l"(cc) : "f"(c));
#pragma unroll
    for (int i = 0; i < kChains; ++i) {
        const float x = (float)(threadIdx.x + i);
        asm("mov.b64 %0, {%1, %1};" : "=l"(a[i]) : "f"(x));
    }
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < kChains; ++i) asm volatile("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(a[i]) : "l"(bb), "l"(cc));
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kChains; ++i) {
        float lo, hi;
        asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(a[i]));
        s += lo + hi;
    }
    if (s == 1234.5f) sink[blockIdx.x] = s;
}

}  // namespace

extern "C" {

// FP32 fma throughput of the current device in TFLOP/s (one fma = 2 flops):
// packed = 0 times fma.rn.f32, packed = 1 fma.rn.f32x2.  Runs `reps` timed
// launches (after one warm-up launch) on `stream` and synchronises it.
// sink: device memory of at least (SMs * 8) floats, never written for the
// inputs used here.  Returns 0 and *tflops on success, -1 on a CUDA error.
int gdn_probe_fp32_tflops(int packed, int reps, float* sink, double* tflops, void* stream)
{
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int dev = 0, sms = 0;
    if (tflops == nullptr || sink == nullptr || reps < 1) return -1;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return -1;
    const int iters = 4096;
    const unsigned grid = (unsigned)(sms * kCtasPerSm);
    cudaEvent_t e0, e1;
    if (cudaEventCreate(&e0) != cudaSuccess) return -1;
    if (cudaEventCreate(&e1) != cudaSuccess) {
        cudaEventDestroy(e0);
        return -1;
    }
    auto launch = [&] {
        if (packed) k_probe_ffma2<<<grid, kThreads, 0, s>>>(iters, 0.999f, 1e-3f, sink);
        else k_probe_ffma<<<grid, kThreads, 0, s>>>(iters, 0.999f, 1e-3f, sink);
    };
    launch();
    cudaEventRecord(e0, s);
    for (int r = 0; r < reps; ++r) launch();
    cudaEventRecord(e1, s);
    float ms = 0.f;
    const bool ok = cudaGetLastError() == cudaSuccess && cudaEventSynchronize(e1) == cudaSuccess &&
                    cudaEventElapsedTime(&ms, e0, e1) == cudaSuccess && ms > 0.f;
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    if (!ok) return -1;
    const double lanes = packed ? 2.0 : 1.0;
    const double flops = 2.0 * lanes * kChains * (double)iters * kThreads * grid * reps;
    *tflops = flops / (ms * 1e-3) / 1e12;
    return 0;
}

}  // extern "C"
