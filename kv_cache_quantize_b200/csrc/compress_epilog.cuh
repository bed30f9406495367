// compress_epilog.cuh -- kv_compress_epilog kernel (aclnnKvCompressEpilog,
// 计算公式 scenarios 1-3 and 约束说明 for the packed-row size).
//
// Work decomposition.  A row of d bf16 values is d/64 SEGMENTS of 64 values:
// the (d-64)/64 nope segments and the rope segment last.  A segment is handled
// by a TEAM of 8 lanes, each lane one 16-byte chunk of 8 values, so a warp
// works on 4 segments at a time and a 64-value quantisation group is one team
// (FP4 groups of 32 / 16 are 4 / 2 lanes of it).  A warp owns a tile of 8
// consecutive rows: lanes 0..7 load the tile's 8 slots once (coalesced), the
// teams walk the tile's segments, and CE_UNROLL segments per team are loaded
// before any is processed so each lane keeps several 16-byte loads in flight.
// Group maxima are butterfly shuffles inside the team.  Every output byte of a
// row has exactly one writer: codes by their chunk's lane, a group's scale by
// the group's first lane, the rope and the zero padding by the rope team.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

struct CompressArgs {
    const uint16_t* x;      // bf16 bit patterns
    int64_t x_row_stride;   // elements
    int64_t T;              // rows
    const void* slots;      // int32 or int64
    int32_t slots_i64;
    PagedRows cache;
    int32_t nseg;           // d / 64 (the last segment is the rope)
    int32_t n;              // d - 64 nope columns
    int32_t concat;         // payload bytes before the zero padding
    int32_t col;            // kvCacheCol
    float x_scale;          // mode 2 rope multiplier
    int32_t x_vec;          // every row chunk is 16-byte aligned
};

constexpr int CE_TILE = 8;
constexpr int CE_UNROLL = 3;
constexpr int CE_THREADS = 256;

__device__ __forceinline__ uint4 ld_scalar8(const uint16_t* p) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = (uint32_t)__ldcs(p + 2 * i) | ((uint32_t)__ldcs(p + 2 * i + 1) << 16);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ int64_t load_slot(const void* slots, int is64, int64_t i) {
    return is64 ? reinterpret_cast<const int64_t*>(slots)[i] : (int64_t) reinterpret_cast<const int32_t*>(slots)[i];
}

// One segment.  All lanes call this (the shuffles need the whole warp); lanes
// whose segment is inactive or skipped carry live == false.
template <int MODE, int G>
__device__ __forceinline__ void ce_segment(const CompressArgs& a, const uint4& v, bool live, int64_t slot,
                                           int j, int sub) {
    constexpr int GL = (MODE == 2 ? G : 64) / 8;   // lanes per quantisation group
    uint32_t m = absmax_bits8(v);
    if (GL >= 2) m = max(m, __shfl_xor_sync(FULL_MASK, m, 1));
    if (GL >= 4) m = max(m, __shfl_xor_sync(FULL_MASK, m, 2));
    if (GL >= 8) m = max(m, __shfl_xor_sync(FULL_MASK, m, 4));
    if (!live) return;

    uint8_t* row = slot_row(a.cache, slot);
    const bool rope = (j == a.nseg - 1);
    float f[8];
    widen8<false>(v, f);
    const float amax = __uint_as_float(m << 16);

    if (MODE == 0) {
        if (!rope) {
            // scale_g = amax / FP8_MAX, stored as bf16; codes use the stored scale
            const uint32_t sb = to_bf16_bits(__fdiv_rn(amax, 448.0f));
            const float sf = __uint_as_float(sb << 16);
            uint2 codes = make_uint2(0u, 0u);
            if (sf != 0.0f) {
                float q[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(f[i], sf);
                codes = fp8x8<false>(q);
            }
            st_b64(row + j * 64 + sub * 8, codes);
            if (sub == 0) st_b16(row + a.n + 128 + 2 * j, sb);
        } else {
            st_b128(row + a.n + sub * 16, v);
            for (int p = a.concat + sub; p < a.col; p += 8) row[p] = 0;
        }
    } else if (MODE == 1) {
        if (!rope) {
            // E8M0 scale: amax / FP8_MAX rounded up to a power of two
            const uint32_t b = e8m0_ceil(__fdiv_rn(amax, 448.0f));
            const float mul = e8m0_reciprocal(b);
            float q[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(f[i], mul);
            st_b64(row + j * 64 + sub * 8, fp8x8<false>(q));
            if (sub == 0) st_b8(row + a.n + 128 + j, b);
        } else {
            st_b128(row + a.n + sub * 16, v);
        }
    } else {
        if (!rope) {
            // FP4 E2M1 per group of G, bf16 scale = amax / 6
            const uint32_t sb = to_bf16_bits(__fdiv_rn(amax, 6.0f));
            const float sf = __uint_as_float(sb << 16);
            uint32_t codes = 0u;
            if (sf != 0.0f) {
                float q[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(f[i], sf);
                codes = e2m1x8(q);
            }
            st_b32(row + j * 32 + sub * 4, codes);
            if (sub % GL == 0) st_b16(row + a.n / 2 + 64 + 2 * (j * (64 / G) + sub / GL), sb);
        } else {
            // static rope: FP8 E4M3 of x * xScale
            float q[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(f[i], a.x_scale);
            st_b64(row + a.n / 2 + sub * 8, fp8x8<false>(q));
            for (int p = a.concat + sub; p < a.col; p += 8) row[p] = 0;
        }
    }
}

template <int MODE, int G>
__global__ void __launch_bounds__(CE_THREADS) compress_epilog_kernel(const CompressArgs a) {
    const int lane = threadIdx.x & 31;
    const int team = lane >> 3;
    const int sub = lane & 7;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t ntiles = (a.T + CE_TILE - 1) / CE_TILE;

    for (int64_t tile = gwarp; tile < ntiles; tile += nwarps) {
        const int64_t row0 = tile * CE_TILE;
        const int rows = (int)(a.T - row0 < CE_TILE ? a.T - row0 : CE_TILE);
        int64_t my_slot = -1;
        if (lane < rows) {
            my_slot = load_slot(a.slots, a.slots_i64, row0 + lane);
            if (my_slot != -1 && !slot_ok(my_slot, a.cache.num_slots)) {
                raise_fault(FAULT_SLOT_RANGE);
                my_slot = -1;
            }
        }
        const int nsegs = rows * a.nseg;
        for (int s0 = 0; s0 < nsegs; s0 += 4 * CE_UNROLL) {
            uint4 v[CE_UNROLL];
            int64_t sl[CE_UNROLL];
            int jj[CE_UNROLL];
            bool live[CE_UNROLL];
#pragma unroll
            for (int u = 0; u < CE_UNROLL; ++u) {
                const int seg = s0 + 4 * u + team;
                const bool act = seg < nsegs;
                const int r = act ? seg / a.nseg : 0;
                jj[u] = seg - r * a.nseg;
                sl[u] = __shfl_sync(FULL_MASK, my_slot, r);
                live[u] = act && sl[u] >= 0;
                v[u] = make_uint4(0u, 0u, 0u, 0u);
                if (live[u]) {
                    const uint16_t* p = a.x + (row0 + r) * a.x_row_stride + jj[u] * 64 + sub * 8;
                    v[u] = a.x_vec ? ld_stream16(p) : ld_scalar8(p);
                }
            }
#pragma unroll
            for (int u = 0; u < CE_UNROLL; ++u) ce_segment<MODE, G>(a, v[u], live[u], sl[u], jj[u], sub);
        }
    }
}

}  // namespace kvq
