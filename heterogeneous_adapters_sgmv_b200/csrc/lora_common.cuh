// Device-side building blocks shared by the LoRA kernels (sm_100a only): adapter
// descriptors, bf16 <-> fp32 helpers, mbarriers, bulk async copies, cluster shared memory,
// programmatic dependent launch, and bounded waits that report instead of hanging.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lora_sgmv.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a (B200) only"
#endif

namespace lora {

// One adapter of a table, as the kernels see it.
struct __align__(32) AdapterDesc {
    const void *A;        // [rank, h] row-major
    const void *B;        // [o, rank] row-major
    int32_t rank;
    float scale;
    const float *sigma;   // three-stage form: Sigma_i (rank x rank or rank values, fp32), else null
};
static_assert(sizeof(AdapterDesc) == 32, "descriptor size");

// Default upper bound of a bounded wait: about two seconds of %globaltimer.  Kernels take the
// bound from their parameters (option "wait_limit_ns"), so a test can shorten it.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Round-to-nearest-even fp32 -> bf16 of a pair, packed low half first.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}

// ---------------------------------------------------------------------------------------
// mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init_cluster()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// Arrive on the barrier at the same smem offset in cluster CTA `rank` (release, cluster scope).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar, uint32_t rank)
{
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(bar), "r"(rank));
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote)
                 : "memory");
}

// One bounded-time probe of a phase.  The suspend-time hint lets the hardware park the thread
// until the phase completes (or ~0.5 ms pass) instead of spinning, so waiting warps do not take
// issue slots from the warps that are working.
constexpr uint32_t kSuspendHintNs = 500000u;

// Arrive on a peer's barrier without release semantics: for signals whose preceding accesses
// are loads whose values have already been consumed (nothing left to order), this avoids a
// cluster-scope fence behind unrelated outstanding stores.
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t bar, uint32_t rank)
{
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(bar), "r"(rank));
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// Bounded waits: false after `limit_ns` of %globaltimer, with LORA_STATUS_TIMEOUT latched into
// *status.  The fast path (phase already complete) is inlined; the polling loop is a separate
// function so the hot code stays small (instruction-cache misses dominate short kernels).
// Between probes the warp sleeps (32 ns doubling to 512 ns), so waiting warps do not take issue
// slots from the warps that are working, and the clock is read only once per probe.
static __device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, uint32_t *status, bool cluster,
                                                   uint64_t limit_ns)
{
    const uint64_t t0 = globaltimer_ns();
    uint32_t pause = 32;
    for (;;) {
        if (cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
        __nanosleep(pause);
        pause = pause < 512 ? 2 * pause : 512;
        if (globaltimer_ns() - t0 > limit_ns) {
            atomicOr(status, LORA_STATUS_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t *status, uint64_t limit_ns)
{
    return mbar_try_wait(bar, parity) || mbar_wait_slow(bar, parity, status, false, limit_ns);
}

__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, uint32_t *status,
                                                  uint64_t limit_ns)
{
    return mbar_try_wait_cluster(bar, parity) || mbar_wait_slow(bar, parity, status, true, limit_ns);
}

// ---------------------------------------------------------------------------------------
// bulk async copies (TMA engine, untiled, no multicast)

// global -> this CTA's shared memory; completion counted in bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}


// 2-D tiled TMA load (no multicast) of box {c0, c1} of `tmap` into this CTA's shared memory.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, int32_t c0, int32_t c1, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(tmap), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// 2-D tiled TMA store of box {c0, c1} of `tmap` from this CTA's shared memory (bulk group).
// The innermost coordinate times the element size must be a multiple of 16 bytes and no
// coordinate may be negative.
__device__ __forceinline__ void tma_store_2d(const void *tmap, uint32_t src, int32_t c0, int32_t c1)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(tmap),
                 "r"(c0), "r"(c1), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk group has finished reading its shared-memory source.
__device__ __forceinline__ void bulk_wait_group_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until at most the newest committed bulk group may still be reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// Wait until every committed bulk group has completed (its writes performed).
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Hint: bring a 128-byte line into L2.
__device__ __forceinline__ void prefetch_l2(const void *p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Hint: bring a 128-byte line into this SM's L1.
__device__ __forceinline__ void prefetch_l1(const void *p)
{
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// Asynchronous store of 16 bytes into cluster CTA `rank`'s shared memory at the same offset as
// `local_addr`; completion is counted in bytes on that CTA's mbarrier at offset `local_bar`.
__device__ __forceinline__ void st_async_v4(uint32_t local_addr, uint32_t local_bar, uint32_t rank, float4 v)
{
    uint32_t ra, rb;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(local_addr), "r"(rank));
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rb) : "r"(local_bar), "r"(rank));
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(ra),
                 "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(rb)
                 : "memory");
}

// ---------------------------------------------------------------------------------------
// cluster

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_id_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t nclusters_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

// Split cluster barrier: arrive (relaxed; pair with an explicit release fence when needed)
// now, wait (acquire) later, so the barrier latency hides behind independent work.
__device__ __forceinline__ void cluster_arrive_relaxed()
{
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire()
{
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Bring a TMA tensor map into the descriptor cache ahead of its first use.
__device__ __forceinline__ void prefetch_tensormap(const void *p)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(p) : "memory");
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Loads from a peer CTA's shared memory.  No memory clobber: callers order them after the
// acquiring wait that made the peer's data visible, and independent loads stay in flight together.
__device__ __forceinline__ float ld_dsmem_f32(uint32_t local_addr, uint32_t rank)
{
    uint32_t remote;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote));
    return v;
}

__device__ __forceinline__ float4 ld_dsmem_f32x4(uint32_t local_addr, uint32_t rank)
{
    uint32_t remote;
    float4 v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(remote));
    return v;
}

// Named barrier over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier over `count` threads that also returns the AND of `pred` over them: used so a
// bounded wait that ran out in any thread stops all of them at the same point.
__device__ __forceinline__ bool named_bar_and(uint32_t id, uint32_t count, bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n"
        " setp.ne.u32 p, %1, 0;\n"
        " bar.red.and.pred q, %2, %3, p;\n"
        " selp.u32 %0, 1, 0, q;\n}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// ---------------------------------------------------------------------------------------
// programmatic dependent launch

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------------------
// optional phase tracing (compiled in only with -DLORA_TRACE): per-CTA clock64 marks

#ifdef LORA_TRACE
constexpr int kTraceCtas = 4096;
constexpr int kTraceSlots = 64;
// defined (once) by the translation unit that uses the marks
#define LORA_TRACE_MARK(slot)                                                              \
    do {                                                                                   \
        if (blockIdx.x < (unsigned)::lora::kTraceCtas)                                     \
            ::lora::lora_trace_buf[blockIdx.x * ::lora::kTraceSlots + (slot)] = clock64(); \
    } while (0)
#else
#define LORA_TRACE_MARK(slot) \
    do {                      \
    } while (0)
#endif

}  // namespace lora
