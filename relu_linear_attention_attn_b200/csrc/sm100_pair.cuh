// sm_100a building blocks for UMMAs spread over a pair of SMs (a cluster of two
// CTAs, tcgen05 cta_group::2): loads that complete on the pair leader's mbarrier,
// the pair UMMA, its commits, and the remote arrives and polling waits of the
// hand-offs between the two CTAs.  Each CTA loads only into its own shared memory
// (no multicast load).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100_primitives.cuh"

namespace sana {

// TMA load into this CTA's shared memory whose bytes complete on the pair leader's
// mbarrier (a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* m,
                                                 uint32_t leader_bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(m), "r"(leader_bar), "r"(x), "r"(y)
        : "memory");
}

// D[tmem] (+)= A * B^T over the pair (M = 256), issued by the leader alone.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5, %5, %5, %5, %5}, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u), "r"(0u)
        : "memory");
}

// Arrive once on the leader's own mbarrier when its pair UMMAs so far are complete.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// The same, arriving on the barrier at this offset in both CTAs of the pair (CTA
// mask 0b11).  This is the commit's own signal, not a data copy.
__device__ __forceinline__ void umma_commit_both(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"((uint16_t)3)
        : "memory");
}

// Wait for a phase by polling (no suspension, so a hand-off on the critical path
// costs no wake-up), giving up after `limit_ns` as mbar_wait does.
__device__ __forceinline__ bool mbar_wait_spin(uint64_t* bar, uint32_t parity, int site,
                                               uint64_t limit_ns = 2000000000ull) {
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_test(bar, parity)) return true;
        if (global_timer_ns() - t0 > limit_ns) {
            record_error(kErrWaitTimeout, site);
            return false;
        }
    }
}

// Arrive on an mbarrier of another CTA of the cluster (release at cluster scope).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* m,
                                                 uint32_t leader_bar, int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(m), "r"(leader_bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// TMEM allocation, relinquish and release for a pair: one warp of each CTA (the
// same warp index in both) executes each of them.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

}  // namespace sana
