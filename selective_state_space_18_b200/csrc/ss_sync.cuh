// ss_sync.cuh -- synchronisation primitives of the scan kernel, all with bounded waits.
//
//  * mbarriers in shared memory between the IO warp and the scan warps of a CTA;
//  * epoch-tagged flags in global memory that pass the scan carry from one
//    sequence segment to the next (possibly on another SM);
//  * a work counter in global memory handing out (channel group, segment) units.
//
// Every wait gives up after a fixed time (2 s, measured with the global timer),
// records SS_ERR_TIMEOUT in the status word and lets the caller unwind; nothing here
// can spin forever.
#pragma once

#include <cuda.h> // CUtensorMap
#include <cuda_runtime.h>
#include <stdint.h>

namespace ss {

constexpr uint64_t kWaitLimitNs = 2000000000ull; // 2 s: far above any legitimate wait
constexpr uint32_t kStatusTimeout = 7u;          // SS_ERR_TIMEOUT

// Time limit override for the waits of later calls, in microseconds (0: kWaitLimitNs).
// Lets a test make a wait run out quickly; set through ss_debug_set_wait_limit.
__device__ uint32_t g_ss_wait_limit_us;

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint64_t wait_limit_ns(bool overridable)
{
    const uint32_t us = overridable ? *reinterpret_cast<volatile uint32_t *>(&g_ss_wait_limit_us) : 0u;
    return us ? uint64_t(us) * 1000ull : kWaitLimitNs;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

// Arrive once and announce `bytes` of asynchronous (TMA) writes the phase must also
// wait for.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// 2-D tile load global -> this CTA's shared memory through a tensor map, completing
// on `bar` (tile mode, no multicast; the tensor map decides the swizzle: none for the
// x and dt tiles, a span of one tile row for the B and C tiles).  c0 is the innermost
// (contiguous) coordinate.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int32_t c0, int32_t c1,
                                            uint64_t *bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
                 : "memory");
}

// Prefetch a 2-D tile into L2 through a tensor map (nothing is written to shared
// memory and nothing is waited for): a later plain load of the tile then hits L2.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *map, int32_t c0, int32_t c1)
{
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1)
                 : "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before later
// asynchronous-proxy (TMA) writes to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// One test of the phase.  If it has not completed, the thread may wait in hardware
// for a short, system-defined time before the test returns false.  (An explicit
// suspend-time hint was measured to resume waiting warps later than this form.)
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return ok != 0;
}

// Wait until the phase of `bar` with the given parity has completed.  Returns false
// (after recording a timeout in *status) if it did not within the time limit.  A NULL
// status marks a drain wait (for copies in flight), which keeps the default limit
// whatever the override says.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t *status)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t limit = wait_limit_ns(status != nullptr);
    const uint64_t t0 = global_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity))
            return true;
        if (global_ns() - t0 > limit)
            break;
    }
    if (status)
        atomicOr(status, 1u << kStatusTimeout);
    return false;
}

__device__ __forceinline__ uint64_t ld_acquire_gpu(const uint64_t *p)
{
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(uint64_t *p, uint64_t v)
{
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// All lanes of a warp poll `flag` until it holds `want`.  Returns false on timeout.
__device__ __forceinline__ bool flag_wait(const uint64_t *flag, uint64_t want, uint32_t *status)
{
    const uint64_t limit = wait_limit_ns(true);
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0;; ++i) {
        if (ld_acquire_gpu(flag) == want)
            return true;
        if (global_ns() - t0 > limit)
            break;
        __nanosleep(i < 64 ? 32 : 256);
    }
    if (status)
        atomicOr(status, 1u << kStatusTimeout);
    return false;
}

// Next work unit of this call: one fetch-and-add on the work counter (the last
// warp of the call resets it to 0, so every call starts from unit 0).
__device__ __forceinline__ uint32_t grab_unit(uint32_t *counter)
{
    return atomicAdd(counter, 1u);
}

} // namespace ss
