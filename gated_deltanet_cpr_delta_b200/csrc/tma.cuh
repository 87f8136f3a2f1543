// tma.cuh -- tensor-memory-accelerator (TMA) tile loads into shared memory (sm_100a).
//
// A [T, H, D] token tensor (q, k or v) is described to the TMA unit as a 3-D
// tensor (D innermost, then H, then T) and a box of D x 1 x n tokens: one
// cp.async.bulk.tensor copies n consecutive tokens of one head into a dense
// [n][D] tile in shared memory and signals an mbarrier with the byte count.
// Boxes that reach past the last token are zero-filled by the hardware.  Every
// copy here starts at x = 0 (the 16-byte rule on the innermost coordinate) and
// uses no cluster multicast; the tensor maps only ever cover this GPU's own
// memory.
#pragma once

#include <cuda.h>

#include "schedule.cuh"

namespace gdn {

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init_cta(uint64_t* mbar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(mbar)), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Arrive on the mbarrier and announce `bytes` of transaction (the TMA copies
// that complete this phase).
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* mbar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(mbar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_test_parity(uint64_t* mbar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P1;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, P1;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(mbar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity; false once `limit` clocks passed.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* mbar, uint32_t parity, long long limit)
{
    const long long t0 = clock64();
    while (!mbar_test_parity(mbar, parity))
        if (clock64() - t0 > limit) return false;
    return true;
}

// Tokens [tok, tok + box) of head h of the tensor behind `map` -> dst (dense
// [box][D] tile, 128-byte aligned), completing on mbar.
__device__ __forceinline__ void tma_load_tokens(void* dst, const CUtensorMap* map, int h, int tok, uint64_t* mbar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(h), "r"(tok), "r"(smem_addr(mbar))
        : "memory");
}

// Generic-proxy accesses of shared memory before this point are ordered before
// later async-proxy (TMA) writes to it.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

}  // namespace gdn
