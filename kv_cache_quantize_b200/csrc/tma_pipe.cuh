// tma_pipe.cuh -- shared-memory staging with the Blackwell bulk-copy engine.
//
// A producer warp moves input rows from HBM into a ring of shared-memory
// stages with cp.async.bulk (1-D TMA, one copy per row, completion counted in
// bytes on the stage's "full" mbarrier); consumer warps wait on "full", work
// on the stage and release it on the stage's "empty" mbarrier.  No cluster
// multicast is used: every copy reads this GPU's own memory into this CTA.
//
// Every wait is bounded: after PIPE_WAIT_LIMIT unsuccessful try_wait calls the
// waiter sets FAULT_TIMEOUT in the device fault word and gives up, so a logic
// error cannot hang the GPU.
#pragma once

#include <cstdint>

#include "kvq_device.cuh"

namespace kvq {

constexpr unsigned FAULT_TIMEOUT = 0x2u;
constexpr uint32_t PIPE_WAIT_LIMIT = 1u << 22;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// make the initialised barriers visible to the bulk-copy (async) proxy
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait until the phase of the given parity has completed; false (and the
// FAULT_TIMEOUT bit) after `limit` unsuccessful tries.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit = PIPE_WAIT_LIMIT) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    raise_fault(FAULT_TIMEOUT);
    return false;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait until the phase of the given parity has completed; false (and the
// FAULT_TIMEOUT bit) once about `ns` nanoseconds have passed without it.  For
// waits whose legitimate length varies with the problem (a whole GEMM main
// loop), where a bound in tries would be either too short or far too long.
__device__ __forceinline__ bool mbar_wait_ns(uint64_t* bar, uint32_t parity, uint64_t ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > ns) break;
    }
    raise_fault(FAULT_TIMEOUT);
    return false;
}

// 1-D bulk copy HBM -> this CTA's shared memory.  dst, src 16-byte aligned,
// bytes a multiple of 16; completion is counted on bar.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 1-D bulk copy this CTA's shared memory -> global (a bulk async-group).
// dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_s2g(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// all committed bulk stores of this thread have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// all committed bulk stores of this thread are complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// order this thread's generic-proxy shared-memory writes before later
// async-proxy (bulk copy) reads of them
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// barrier over the first `threads` threads of the CTA (named barrier 1)
__device__ __forceinline__ void named_barrier_sync(int threads) {
    asm volatile("bar.sync 1, %0;" ::"r"(threads) : "memory");
}

// arrive at named barrier 1 without waiting
__device__ __forceinline__ void named_barrier_arrive(int threads) {
    asm volatile("bar.arrive 1, %0;" ::"r"(threads) : "memory");
}

}  // namespace kvq
