// ptx.cuh -- thin inline-PTX wrappers used by the libselscan kernels
// (sm_100a): mbarriers, bulk tensor copies (TMA, no multicast), proxy
// fences, named barriers, gpu-scope acquire/release flags and the fast
// special-function instructions.  Every spin built on these is bounded by a
// time limit measured on %globaltimer (mbar_wait, spin_flag).
#pragma once

#include <cstdint>
#include <cuda.h>

namespace selscan {

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;"
                 :: "r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(smem_addr(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];"
                 :: "r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// try_wait that lets the hardware suspend the thread until the phase
// completes or `hint_ns` nanoseconds pass, instead of returning at once: a
// waiting warp then issues no instructions (a polling loop would take issue
// slots from the warps that share its scheduler).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity,
                                                    uint32_t hint_ns)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns) : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, giving up after
// `timeout_ns` nanoseconds (%globaltimer).  Returns false on time-out.  The
// fast path is a bare try_wait; after that the thread sleeps in the
// hardware between checks (at most 20 us at a time) and reads the timer
// after each wake-up.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          uint64_t timeout_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t start = global_timer_ns();
    while (!mbar_try_wait_sleep(bar, parity, 20000u)) {
        if (global_timer_ns() - start > timeout_ns)
            return false;
    }
    return true;
}

// Wait for a slow event (the producer waiting for a stage to be released):
// poll with a short sleep between tries, so that the waiting warp takes
// almost no issue slots from the warps that share its scheduler.  Returns
// false after `timeout_ns`.
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t *bar, uint32_t parity,
                                                  uint64_t timeout_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t start = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        __nanosleep(200);
        if (global_timer_ns() - start > timeout_ns)
            return false;
    }
    return true;
}

// ---------------------------------------------------- bulk tensor copies
// Tiled loads complete on an mbarrier (complete_tx); stores go through the
// bulk async-group mechanism.  The innermost coordinate c0 must be a
// multiple of 16 bytes' worth of elements (callers pass chunk-aligned t).
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map,
                                            uint64_t *bar, int c0, int c1, int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        :: "r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)),
           "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map,
                                             const void *src, int c0, int c1, int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
        :: "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(src)),
           "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void bulk_commit()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" :: "n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait_all()
{
    asm volatile("cp.async.bulk.wait_group %0;" :: "n"(N) : "memory");
}

// generic-proxy shared-memory writes -> later async-proxy (TMA) reads
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];"
                 :: "l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------- named barriers
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads)
{
    asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(nthreads) : "memory");
}

// Barrier over `nthreads` threads that also ORs a predicate across them, so
// that a group can agree on leaving a loop at the same iteration.
__device__ __forceinline__ bool named_bar_any(uint32_t id, uint32_t nthreads, bool pred)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred pi, po;\n\t"
                 "setp.ne.u32 pi, %1, 0;\n\t"
                 "bar.red.or.pred po, %2, %3, pi;\n\t"
                 "selp.u32 %0, 1, 0, po;\n\t}"
                 : "=r"(r) : "r"(uint32_t(pred)), "r"(id), "r"(nthreads) : "memory");
    return r != 0;
}

// ------------------------------------------------ gpu-scope flag access
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(uint32_t *p, uint32_t v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

// Spin until *flag == want or `timeout_ns` passes; false on time-out.
__device__ __forceinline__ bool spin_flag(const uint32_t *flag, uint32_t want,
                                          uint64_t timeout_ns)
{
    if (ld_acquire_gpu(flag) == want)
        return true;
    const uint64_t start = global_timer_ns();
    uint32_t spins = 0;
    while (ld_acquire_gpu(flag) != want) {
        if ((++spins & 63u) == 0u) {
            if (global_timer_ns() - start > timeout_ns)
                return false;
            __nanosleep(64);
        }
    }
    return true;
}

// ------------------------------------------- asynchronous 16-byte copies
// global -> shared, `src_bytes` (0..16) read and the rest of the 16 bytes
// zero-filled; completion tracked per thread by commit / wait groups.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 :: "r"(smem_addr(smem_dst)), "l"(gsrc), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory");
}

// ------------------------------------------- fast special functions
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float lg2_approx(float x)
{
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// tanh on the special-function unit (maximum absolute error about 2^-11)
__device__ __forceinline__ float tanh_approx(float x)
{
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp_approx(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace selscan
