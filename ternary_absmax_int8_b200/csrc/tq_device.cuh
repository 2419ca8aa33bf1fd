// tq_device.cuh -- device-side building blocks shared by libtq's kernels:
// mbarriers with bounded waits, 1-D bulk copies (TMA engine, no multicast),
// programmatic-dependent-launch controls and the mixed-sign dp4a.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace tq {

// Kernels report errors by OR-ing bits into the library's device error word
// (defined in tq_api.cu, read and cleared by tq_device_error()); its address
// reaches them through their launch parameters.
constexpr unsigned kErrWaitTimeout = 1u;  // a bounded pipeline wait gave up

// A pipeline wait that has not completed after this many nanoseconds of
// global time gives up: it sets the error word and the kernel winds down.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Make mbarrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase with the given parity has completed. Returns false
// (after recording kErrWaitTimeout in *err) if it does not complete within
// limit_ns nanoseconds of global time.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, unsigned *err,
                                          unsigned long long limit_ns = kWaitLimitNs)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((i & 255u) == 0 && global_ns() - t0 > limit_ns) {
            atomicOr(err, kErrWaitTimeout);
            return false;
        }
    }
}

// mbar_wait for all 32 lanes of a warp together, with a warp-uniform result
// (so that a timeout can never split a warp).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity, unsigned *err)
{
    bool done = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, done))
        return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        done = done || mbar_try_wait(bar, parity);
        if (__all_sync(0xffffffffu, done))
            return true;
        if ((i & 255u) == 0) {
            const bool late = global_ns() - t0 > kWaitLimitNs;
            if (__any_sync(0xffffffffu, late)) {
                if ((threadIdx.x & 31) == 0)
                    atomicOr(err, kErrWaitTimeout);
                return false;
            }
        }
    }
}

// 1-D bulk copy global -> shared through the TMA engine; completion is
// reported to `bar` as transaction bytes. dst, src 16-byte aligned; bytes a
// multiple of 16. `policy` is an L2 cache policy from createpolicy.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Programmatic dependent launch: wait for the grids this one depends on
// (no-op when launched without the attribute) / let dependents launch.
__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Named barrier over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Four-way dot product of unsigned bytes a (codes, possibly shifted left by
// 2p) with signed bytes b (int8 activations), added to c.
__device__ __forceinline__ int32_t dp4a_us(uint32_t a, uint32_t b, int32_t c)
{
    int32_t d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint4 lds128(const void *p)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

}  // namespace tq
