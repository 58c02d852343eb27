// cluster.cuh -- thread-block clusters (sm_90+, used on sm_100a): the CTAs of
// a cluster run at the same time, read one another's shared memory
// (distributed shared memory) and meet at a hardware barrier.  The forward's
// small-problem path passes each Newton iteration's tile aggregates this way,
// with no round trip through L2 and no polling.  Only plain loads of the
// cluster's own shared memory are used (no TMA, no multicast).
#pragma once

#include <stdint.h>

#include "tma.cuh"

namespace pararnn {

// this CTA's rank in its cluster (0 .. cluster size - 1)
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Every thread of every CTA of the cluster arrives, then waits: shared-memory
// writes before the arrive are visible to reads from any CTA of the cluster
// after the wait.  Like __syncthreads, every thread must take the same number
// of these barriers (the hardware holds the cluster's CTAs resident together,
// so the barrier always completes).
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
// arrive without release: for threads that publish nothing to other CTAs
// (their own CTA's reads are ordered by block barriers), so the arrive
// waits for none of their outstanding memory operations
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive, with release at cluster scope, on the mbarrier at the same
// shared-memory offset as `local_bar` in the CTA of rank `rank`: the
// calling thread's earlier writes are visible to a thread of that CTA that
// sees the barrier's phase complete with cluster-scope acquire.
__device__ __forceinline__ void mbar_arrive_remote(uint64_t* local_bar, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local_bar)), "r"(rank));
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}

// mbarrier_try_wait with cluster-scope acquire (the arrivals came from other
// CTAs of the cluster)
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void fence_acq_rel_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

// a float at the same shared-memory offset as `local` in the CTA of rank `rank`
__device__ __forceinline__ float ld_dsmem(const float* local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// Status flags of a call whose workspace header is not cleared before it
// runs (the small-problem path launches nothing but its kernel): a 64-bit
// word {call number, flags}; a flag set by this call replaces the flags of
// an older call.
__device__ __forceinline__ void set_tagged_status(unsigned long long* word, uint32_t epoch, unsigned bit) {
    unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(word);
    while (true) {
        const unsigned long long want = (static_cast<uint32_t>(old >> 32) == epoch)
                                            ? (old | bit)
                                            : ((static_cast<unsigned long long>(epoch) << 32) | bit);
        if (want == old) return;
        const unsigned long long seen = atomicCAS(word, old, want);
        if (seen == old) return;
        old = seen;
    }
}

}  // namespace pararnn
