// mea_pipe.cuh -- shared-memory barriers and 1-D bulk copies for the
// pipelined kernels (a producer thread streams tiles into a shared-memory
// ring; consumer warps compute from it).
#pragma once

#include <cstdint>

namespace mea {

// ---------------------------------------------------------------- mbarrier
// Shared-memory barriers that 1-D bulk copies (cp.async.bulk) complete.
// Every wait is bounded: after kMbarSpins polls that each suspend for up to
// kMbarSuspendNs it gives up and returns false (the caller records an error
// instead of hanging).

constexpr uint32_t kMbarSpins = 1u << 22;
constexpr uint32_t kMbarSuspendNs = 1000;
// The limit of the bounded-wait self-test (a few milliseconds at most).
constexpr uint32_t kMbarSpinsSelfTest = 1u << 12;

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
// Makes the initialised barriers visible to the async proxy (bulk copies).
__device__ __forceinline__ void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t spins = kMbarSpins)
{
    for (uint32_t i = 0; i < spins; ++i) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done)
            : "r"(bar), "r"(parity), "r"(kMbarSuspendNs)
            : "memory");
        if (done) return true;
    }
    return false;
}
// Global -> shared 1-D bulk copy of `bytes` (a multiple of 16; both addresses
// 16-byte aligned) that completes `bytes` transactions on barrier `bar`.
// The destination is this CTA's own shared memory; no multicast.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
// Named barrier `id` (1..15; 0 is __syncthreads) that completes when
// `threads` threads (a multiple of 32: whole warps) have reached it.
__device__ __forceinline__ void named_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace mea
