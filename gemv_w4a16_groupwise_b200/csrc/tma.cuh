// mbarrier / TMA wrappers (inline PTX, sm_100a) with bounded waits.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace w4 {

// A wait that has not completed after g_wait_limit_ns (2 s unless a test
// shortens it) is abandoned: the kernel records the reason in g_error_word
// and unwinds instead of hanging.

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Test the phase; while it is incomplete the thread may be suspended in
// hardware for up to `suspend_ns` (it resumes as soon as the phase
// completes), so waiting threads do not take issue slots from working ones.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t suspend_ns = 0) {
    uint32_t ok;
    if (suspend_ns == 0) {
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
            " selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
    } else {
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
            " selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity), "r"(suspend_ns)
            : "memory");
    }
    return ok != 0;
}

// Wait for the phase with the given parity to complete.  Returns false (and
// records `err`) when the wait exceeds g_wait_limit_ns or when another role
// of the CTA has already raised *abort; the caller then unwinds.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort, unsigned int err) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long start = global_timer_ns();
    const unsigned long long limit = g_wait_limit_ns;
    for (;;) {
        // suspended for at most 20 us per test, so the abort flag and the
        // time limit are still checked often
        if (mbar_try_wait(bar, parity, 20000u)) return true;
        if (*abort) return false;
        if (global_timer_ns() - start > limit) {
            record_error(err);
            *abort = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled TMA load into this CTA's shared memory, completing on `bar`.
// c0 is the innermost (contiguous) coordinate in elements; c0 * elem_size
// must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// One elected lane of the warp orders the warp's earlier shared-memory
// reads before the async proxy's writes, arms `bar` for `bytes` and issues
// N (1 or 3) 2-D TMA loads that complete on it.  Every lane computes the
// same operands; only the election is predicated, so the warp does not
// diverge.
template <int N>
__device__ __forceinline__ void tma_issue_elected(uint64_t* bar, uint32_t bytes, void* d0, const CUtensorMap* m0,
                                                  int x0, int y0, void* d1 = nullptr, const CUtensorMap* m1 = nullptr,
                                                  int x1 = 0, int y1 = 0, void* d2 = nullptr,
                                                  const CUtensorMap* m2 = nullptr, int x2 = 0, int y2 = 0) {
    static_assert(N == 1 || N == 3, "N");
    if (N == 1) {
        asm volatile(
            "{\n .reg .pred P;\n elect.sync _|P, 0xffffffff;\n"
            " @P fence.proxy.async.shared::cta;\n"
            " @P mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n"
            " @P cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%2], [%3, {%4, %5}], [%0];\n}\n" ::"r"(smem_u32(bar)),
            "r"(bytes), "r"(smem_u32(d0)), "l"(reinterpret_cast<uint64_t>(m0)), "r"(x0), "r"(y0)
            : "memory");
    } else {
        asm volatile(
            "{\n .reg .pred P;\n elect.sync _|P, 0xffffffff;\n"
            " @P fence.proxy.async.shared::cta;\n"
            " @P mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n"
            " @P cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%2], [%3, {%4, %5}], [%0];\n"
            " @P cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%6], [%7, {%8, %9}], [%0];\n"
            " @P cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%10], [%11, {%12, %13}], [%0];\n}\n" ::"r"(smem_u32(bar)),
            "r"(bytes), "r"(smem_u32(d0)), "l"(reinterpret_cast<uint64_t>(m0)), "r"(x0), "r"(y0),
            "r"(smem_u32(d1)), "l"(reinterpret_cast<uint64_t>(m1)), "r"(x1), "r"(y1), "r"(smem_u32(d2)),
            "l"(reinterpret_cast<uint64_t>(m2)), "r"(x2), "r"(y2)
            : "memory");
    }
}

// 4-byte cp.async that reads `src_bytes` (0, 2 or 4) and zero-fills the rest.
__device__ __forceinline__ void cp_async_4(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(smem_dst)),
                 "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(src_bytes)
                 : "memory");
}

// Arrive on `bar` once this thread's earlier cp.async copies have landed
// (the arrival is counted in the barrier's initial count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Named barrier over `count` threads (ids 1..15; id 0 is __syncthreads).
__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

}  // namespace w4
