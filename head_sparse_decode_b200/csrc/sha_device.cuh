// sha_device.cuh -- sm_100a building blocks shared by the SHA decode kernels:
// mbarrier pipeline primitives with bounded waits, 1-D bulk async copies
// (global -> shared, completion counted on an mbarrier), dtype conversion,
// and the library's sticky device status word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sha {

// Sticky status bits, read and cleared by sha_get_device_status().
enum : unsigned { kStatusBadIndex = 1u, kStatusTimeout = 2u };

// Sticky device status (one per device per loaded library).
static __device__ unsigned int g_sha_status;

// A pipeline wait that has not completed after this long gives up, raises
// kStatusTimeout and lets the kernel unwind.  Healthy waits last microseconds.
constexpr unsigned long long kWaitLimitNs = 4000000000ull;
// A thread waiting for its own asynchronous copies to land before its block
// exits (or before tensor memory is released) gives up only after this long:
// the copies write into the block's memory, so it waits for them even after
// a pipeline wait has given up.
constexpr unsigned long long kDrainLimitNs = 4000000000ull;

#ifdef SHA_TEST_HOOKS
// Test builds only: the pipeline wait limit is a device variable the tests
// can lower (sha_test_set_wait_limit) to make waits give up on purpose.
static __device__ unsigned long long g_wait_limit_ns = kWaitLimitNs;
__device__ __forceinline__ unsigned long long wait_limit_ns() { return g_wait_limit_ns; }
#else
__device__ __forceinline__ unsigned long long wait_limit_ns() { return kWaitLimitNs; }
#endif

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Make initialised barriers visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// A try_wait may suspend the thread until the phase completes (or a limit of
// the hardware's choosing), so a short wait never reaches the code that gives
// up.  Test builds poll with the non-blocking test_wait instead, so that a
// lowered wait limit makes waits give up; the unwinding is the same code.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
#ifdef SHA_TEST_HOOKS
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
#else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
#endif
    return done != 0;
}

// Wait for the phase of `bar` with the given parity to complete.  Returns
// false (and the caller must unwind) if it has not after wait_limit_ns().
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_timer_ns();
    const unsigned long long limit = wait_limit_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit) return false;
    }
    return true;
}

// mbar_wait for a phase completed by this block's own asynchronous copies
// (or tensor-core work), before their destination is given up: bounded by
// kDrainLimitNs whatever the pipeline limit.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kDrainLimitNs) return false;
    }
    return true;
}

// ---- thread-block clusters --------------------------------------------------
// A unit split across the blocks of one cluster is merged through distributed
// shared memory: each block stores its part of the unit straight into the
// shared memory of the blocks that finish it (asynchronous stores counted on
// their mbarriers), so no block reads another's memory.

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Hardware cluster barrier, split into its two halves.  Every thread of every
// block arrives once; a thread waits before its first access to another
// block's shared memory (its mbarriers must be initialised by then).
__device__ __forceinline__ void cluster_arrive()
{
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait()
{
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Asynchronous stores into the shared memory of block `rank` of this cluster,
// at the same offset as `local` has in this block; the bytes are counted
// (complete_tx) on the mbarrier at `bar`'s offset in that block, so a thread
// there that waits on it sees them.
__device__ __forceinline__ void st_async_f32x2(const float *local, uint32_t rank, float a, float b,
                                               uint64_t *bar)
{
    asm volatile(
        "{\n\t.reg .b32 ra, rb;\n\t"
        "mapa.shared::cluster.u32 ra, %0, %4;\n\t"
        "mapa.shared::cluster.u32 rb, %1, %4;\n\t"
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [ra], {%2, %3}, [rb];\n\t}"
        ::"r"(smem_addr(local)), "r"(smem_addr(bar)), "f"(a), "f"(b), "r"(rank)
        : "memory");
}
__device__ __forceinline__ void st_async_f32(const float *local, uint32_t rank, float a,
                                             uint64_t *bar)
{
    asm volatile(
        "{\n\t.reg .b32 ra, rb;\n\t"
        "mapa.shared::cluster.u32 ra, %0, %3;\n\t"
        "mapa.shared::cluster.u32 rb, %1, %3;\n\t"
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.f32 [ra], %2, [rb];\n\t}"
        ::"r"(smem_addr(local)), "r"(smem_addr(bar)), "f"(a), "r"(rank)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait, with acquire at cluster scope, for a phase completed by other blocks'
// asynchronous stores into this block: what they stored is visible
// afterwards.  The stores write into this block's memory, so the wait is
// bounded by kDrainLimitNs, like a wait for the block's own copies.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const unsigned long long t0 = global_timer_ns();
    while (!mbar_try_wait_cluster(bar, parity)) {
        if (global_timer_ns() - t0 > kDrainLimitNs) return false;
    }
    return true;
}

// The hardware cluster barrier for threads that may be diverged within their
// warp (the kernels' last step under the clustered cut).
__device__ __forceinline__ void cluster_sync_unaligned()
{
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// L2 policy for data read exactly once per call (the selected K/V rows).
__device__ __forceinline__ uint64_t l2_policy_evict_first()
{
    uint64_t policy;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
    return policy;
}

// 1-D bulk async copy global -> this CTA's shared memory; the bytes are
// counted against `bar`'s transaction count.  dst, src 16-byte aligned,
// bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes,
                                              uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// ---- 16-byte asynchronous copies (not through the TMA unit) ---------------------

// Copy 16 bytes global -> shared, bypassing L1; dst and src 16-byte aligned.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint64_t policy)
{
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "l"(policy)
                 : "memory");
}

// The same into the shared address `dst`, reading only src_bytes (16 or 0)
// of src and filling the rest of the 16 bytes with zeros.
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void *src,
                                                 uint32_t src_bytes, uint64_t policy)
{
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(dst),
                 "l"(src), "r"(src_bytes), "l"(policy)
                 : "memory");
}

// Arrive on `bar` (as one of its expected arrivals) once every cp.async this
// thread has issued so far has landed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (bulk copy / TMA) accesses of the same bytes.
__device__ __forceinline__ void fence_proxy_async_shared()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Named barrier over `threads` threads (a multiple of 32), id 1..15.
__device__ __forceinline__ void named_barrier(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---- programmatic dependent launch ------------------------------------------
// A kernel launched with programmatic stream serialization may start while the
// previous kernel in the stream is still running.  pdl_wait() blocks until that
// kernel has completed and its memory is visible (a no-op otherwise): it must
// come before the first read of anything a previous kernel may have written.
// pdl_launch_dependents() lets the next kernel in the stream be scheduled as SMs
// free up.
__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- element conversion ---------------------------------------------------

template <typename T> struct Elem;

template <> struct Elem<__half> {
    static __device__ __forceinline__ float2 pair(uint32_t w)
    {
        __half2 h = *reinterpret_cast<__half2 *>(&w);
        return __half22float2(h);
    }
    static __device__ __forceinline__ __half from_float(float x) { return __float2half_rn(x); }
};

template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float2 pair(uint32_t w)
    {
        __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162 *>(&w);
        return __bfloat1622float2(h);
    }
    static __device__ __forceinline__ __nv_bfloat16 from_float(float x)
    {
        return __float2bfloat16_rn(x);
    }
};

// Two fp32 values rounded to T and packed low/high into one 32-bit register.
template <typename T> __device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi)
{
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Eight 16-bit elements (one 16-byte vector) widened to fp32.
template <typename T>
__device__ __forceinline__ void widen8(const uint4 &v, float (&f)[8])
{
    float2 a = Elem<T>::pair(v.x), b = Elem<T>::pair(v.y);
    float2 c = Elem<T>::pair(v.z), d = Elem<T>::pair(v.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

}  // namespace sha
