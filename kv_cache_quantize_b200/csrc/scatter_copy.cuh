// scatter_copy.cuh -- the memory access pattern of the kv_compress_epilog
// kernels with none of their arithmetic: each valid token's whole input row is
// read (contiguous rows) and the first out_bytes of it are written to the
// token's slot row (scattered rows), skipping -1.  It has no counterpart on the
// pages; it measures what DRAM delivers for this pattern through the same
// engine the pipelined compress kernel uses, the ceiling that kernel is
// compared with.
//
// A CTA is a producer warp and a storer warp around a ring of SB_STAGES stages
// of 32 rows.  The producer loads the tile's slots, keeps the destination row
// pointers beside the stage and brings each valid row in with one 1-D bulk copy
// (global -> shared, completion counted in bytes on the stage's `full`
// mbarrier).  The storer sends each row's first out_bytes out with one bulk
// copy (shared -> global) and releases the stage once the bulk engine has read
// it.  No thread reads or writes the row data itself.
#pragma once

#include "kvq_device.cuh"
#include "tma_pipe.cuh"

namespace kvq {

struct ScatterCopyArgs {
    const uint8_t* x;            // row t starts at x + t * x_row_bytes (16-byte aligned)
    int64_t x_row_bytes;         // row stride in bytes
    int64_t T;
    const void* slots;
    int32_t slots_i64;
    PagedRows cache;             // rows 16-byte aligned
    int32_t in_bytes;            // bytes read per row (a multiple of 16)
    int32_t out_bytes;           // bytes written per row (a multiple of 16, <= in_bytes)
};

constexpr int SB_ROWS = 32;
constexpr int SB_STAGES = 3;
constexpr int SB_THREADS = 64;
constexpr int SB_MAX_ROW_BYTES = 2048;

__host__ __device__ inline uint32_t sb_header_bytes() {
    return ((uint32_t)(16 * SB_STAGES + 8 * SB_STAGES * SB_ROWS) + 127u) & ~127u;
}

__host__ __device__ inline uint32_t sb_smem_bytes(int in_bytes) {
    return sb_header_bytes() + (uint32_t)SB_STAGES * SB_ROWS * (uint32_t)in_bytes;
}

// all but the most recent committed bulk store group of this thread have
// finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all_but_one() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

__global__ void __launch_bounds__(SB_THREADS) scatter_bulk_kernel(const ScatterCopyArgs a) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int S = SB_STAGES;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + S;
    uint8_t** rowptr = reinterpret_cast<uint8_t**>(smem + 16 * S);
    uint8_t* xs = smem + sb_header_bytes();
    const uint32_t pitch = (uint32_t)a.in_bytes;
    const uint32_t stage_bytes = SB_ROWS * pitch;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t ntiles = (a.T + SB_ROWS - 1) / SB_ROWS;

    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
        }
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------- producer ----------------
        auto lane_slot = [&](int64_t tile) -> int64_t {
            const int64_t r = tile * SB_ROWS + lane;
            return (tile < ntiles && r < a.T) ? load_slot(a.slots, a.slots_i64, r) : -1;
        };
        int it = 0;
        int64_t next_slot = lane_slot(blockIdx.x);
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
            const int st = it % S;
            const uint32_t round = (uint32_t)(it / S);
            const int64_t slot = next_slot;
            next_slot = lane_slot(tile + gridDim.x);
            if (!__all_sync(FULL_MASK, mbar_wait(&empty[st], (round & 1u) ^ 1u))) break;
            uint8_t* p = nullptr;
            if (slot != -1) {
                if (slot_ok(slot, a.cache.num_slots)) p = slot_row(a.cache, slot);
                else raise_fault(FAULT_SLOT_RANGE);
            }
            rowptr[st * SB_ROWS + lane] = p;
            const unsigned valid = __ballot_sync(FULL_MASK, p != nullptr);
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(&full[st], (uint32_t)__popc(valid) * pitch);
            __syncwarp();
            if (p != nullptr)
                bulk_copy_g2s(xs + (size_t)st * stage_bytes + (size_t)lane * pitch,
                              a.x + (tile * SB_ROWS + lane) * a.x_row_bytes, pitch, &full[st]);
        }
        // no copy may still be in flight when the CTA exits
        if (lane == 0)
            for (int k = it > S ? it - S : 0; k < it; ++k) mbar_wait(&full[k % S], (uint32_t)(k / S) & 1u);
        return;
    }

    // ---------------- storer ----------------
    int it = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
        const int st = it % S;
        const uint32_t round = (uint32_t)(it / S);
        if (!__all_sync(FULL_MASK, mbar_wait(&full[st], round & 1u))) break;
        uint8_t* p = rowptr[st * SB_ROWS + lane];
        if (p != nullptr) bulk_copy_s2g(p, xs + (size_t)st * stage_bytes + (size_t)lane * pitch, (uint32_t)a.out_bytes);
        bulk_commit();
        if (it > 0) {
            bulk_wait_read_all_but_one();             // tile it-1's rows have left its stage
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[(it - 1) % S]);
        }
    }
    bulk_wait_all();                                  // every store is complete before the CTA exits
}

}  // namespace kvq
