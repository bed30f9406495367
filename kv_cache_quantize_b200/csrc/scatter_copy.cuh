// scatter_copy.cuh -- the memory access pattern of the kv_compress_epilog
// kernels with none of their arithmetic: each valid token's whole input row is
// read (contiguous rows) and the first out_bytes of it are written to the
// token's slot row (scattered rows), skipping -1.  It has no counterpart on the
// pages; it measures what DRAM delivers for this pattern, the ceiling that the
// compress kernels are compared with.
//
// A warp copies two rows per round: lane l loads the 16-byte chunks l, l + 32,
// ... of both rows (streaming loads, nothing allocated in L1) before storing
// any, so a warp keeps up to 2 * NCL * 512 bytes in flight.  Chunks past
// out_bytes are read but not written; they are folded into a per-thread value
// whose only use is a store that happens when it equals a fixed 128-bit
// pattern, which keeps the loads without adding work per chunk.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

struct ScatterCopyArgs {
    const uint8_t* x;            // row t starts at x + t * x_row_bytes (16-byte aligned)
    int64_t x_row_bytes;         // row stride in bytes
    int64_t T;
    const void* slots;
    int32_t slots_i64;
    PagedRows cache;             // rows 16-byte aligned
    int32_t in_chunks;           // bytes read per row / 16
    int32_t out_chunks;          // bytes written per row / 16 (<= in_chunks)
};

constexpr int SC_THREADS = 256;
constexpr int SC_MAX_CHUNKS_PER_LANE = 4;      // rows up to 2048 bytes

__device__ uint4 g_scatter_sink;

__device__ __forceinline__ uint4 ld_nc16(const uint8_t* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

template <int NCL>
__global__ void __launch_bounds__(SC_THREADS) scatter_copy_kernel(const ScatterCopyArgs a) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    uint4 sink = make_uint4(0u, 0u, 0u, 0u);
    for (int64_t r0 = 2 * gwarp; r0 < a.T; r0 += 2 * nwarps) {
        int64_t s[2];
        uint4 v[2][NCL];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t row = r0 + u;
            s[u] = row < a.T ? load_slot(a.slots, a.slots_i64, row) : -1;
            if (s[u] != -1 && !slot_ok(s[u], a.cache.num_slots)) {
                if (lane == 0) raise_fault(FAULT_SLOT_RANGE);
                s[u] = -1;
            }
#pragma unroll
            for (int k = 0; k < NCL; ++k) {
                const int c = lane + 32 * k;
                v[u][k] = (s[u] >= 0 && c < a.in_chunks) ? ld_nc16(a.x + row * a.x_row_bytes + 16 * c)
                                                         : make_uint4(0u, 0u, 0u, 0u);
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (s[u] < 0) continue;
            uint8_t* dst = slot_row(a.cache, s[u]);
#pragma unroll
            for (int k = 0; k < NCL; ++k) {
                const int c = lane + 32 * k;
                if (c < a.out_chunks) {
                    *reinterpret_cast<uint4*>(dst + 16 * c) = v[u][k];
                } else {
                    sink.x ^= v[u][k].x;
                    sink.y ^= v[u][k].y;
                    sink.z ^= v[u][k].z;
                    sink.w ^= v[u][k].w;
                }
            }
        }
    }
    if (sink.x == 0x9e3779b9u && sink.y == 0x7f4a7c15u && sink.z == 0xf39cc060u && sink.w == 0x5cedc834u)
        g_scatter_sink = sink;
}

}  // namespace kvq
