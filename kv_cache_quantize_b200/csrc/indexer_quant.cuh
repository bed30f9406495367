// indexer_quant.cuh -- indexer_quant_cache kernel (indexer_quant_cache,
// 接口功能: mxfp8 / mxfp4 groups of 32 with an E8M0 scale, fp8 one group per
// row with a binary32 scale; 约束说明 for the cache / cache_scale rows).
//
// A row is handled by a TEAM of TEAM lanes (4, 8, 16 or 32), one 16-byte chunk
// of 8 values per lane, so a 32-value group is 4 adjacent lanes and its
// maximum is two butterfly shuffles.  Rows longer than 8*TEAM values (TEAM 32
// only) are walked in blocks of 8*TEAM values.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

struct IndexerArgs {
    const uint16_t* x;
    int64_t x_row_stride;
    int64_t T;
    int32_t d;
    int32_t nchunks;      // ceil(d / 8)
    int32_t x_f16;
    int32_t x_vec;        // every full chunk is 16-byte aligned
    const void* slots;
    int32_t slots_i64;
    PagedRows cache;      // codes
    PagedRows scale;      // cache_scale rows
    int32_t e5m2;         // FP8 codes in E5M2 (else E4M3)
};

constexpr int IX_THREADS = 256;

// Load the values [8c, 8c + 8) of a row, zero beyond d.
__device__ __forceinline__ uint4 ix_load_chunk(const IndexerArgs& a, const uint16_t* xrow, int c) {
    const int nvalid = a.d - 8 * c;
    if (nvalid >= 8 && a.x_vec) return ld_stream16(xrow + 8 * c);
    uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (i < nvalid) w[i >> 1] |= (uint32_t)__ldcs(xrow + 8 * c + i) << (16 * (i & 1));
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void ix_widen(const IndexerArgs& a, const uint4& v, float (&f)[8]) {
    if (a.x_f16) widen8<true>(v, f); else widen8<false>(v, f);
}

__device__ __forceinline__ uint2 ix_fp8x8(const IndexerArgs& a, const float (&q)[8]) {
    return a.e5m2 ? fp8x8<true>(q) : fp8x8<false>(q);
}

__device__ __forceinline__ float ix_amax(const IndexerArgs& a, uint32_t m) {
    return a.x_f16 ? __half2float(__ushort_as_half((unsigned short)m)) : __uint_as_float(m << 16);
}

// mx modes, chunk c of a row (all lanes call it: the scale gather shuffles).
// Group maxima over 4 lanes; the E8M0 bytes of up to four consecutive groups
// are gathered into one 4-byte word written by the first lane of the four.
template <int MODE, int TEAM>
__device__ __forceinline__ void ix_mx_chunk(const IndexerArgs& a, const uint4& v, bool live, uint8_t* crow,
                                            uint8_t* srow, int c, int tl) {
    uint32_t m = absmax_bits8(v);
    m = max(m, __shfl_xor_sync(FULL_MASK, m, 1));
    m = max(m, __shfl_xor_sync(FULL_MASK, m, 2));
    const float fmax = MODE == 3 ? 6.0f : (a.e5m2 ? 57344.0f : 448.0f);
    const uint32_t b = e8m0_ceil(div_by_fmax(ix_amax(a, m), fmax));
    // gather: group g = c / 4 puts its byte at position g % 4 of its word
    uint32_t word = (tl & 3) == 0 ? b << (8 * ((c >> 2) & 3)) : 0u;
    if (TEAM >= 8) word |= __shfl_xor_sync(FULL_MASK, word, 4);
    if (TEAM >= 16) word |= __shfl_xor_sync(FULL_MASK, word, 8);
    const int nvalid = a.d - 8 * c;
    if (!live || nvalid <= 0) return;
    const float mul = e8m0_reciprocal(b);
    float f[8], q[8];
    ix_widen(a, v, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(f[i], mul);
    if (MODE == 0) {
        const uint2 codes = ix_fp8x8(a, q);
        if (nvalid >= 8) st_b64(crow + 8 * c, codes);
        else st_partial(crow + 8 * c, make_uint4(codes.x, codes.y, 0u, 0u), nvalid);
    } else {
        const uint32_t codes = e2m1x8(q);
        if (nvalid >= 8) st_b32(crow + 4 * c, codes);
        else st_partial(crow + 4 * c, make_uint4(codes, 0u, 0u, 0u), (nvalid + 1) / 2);
    }
    if ((c & 15) == 0) {
        // first lane of up to four groups: the word covers groups c/4 .. c/4+3
        const int scol = (a.d + 31) / 32;
        const int g0 = c >> 2;
        const int nb = scol - g0 < 4 ? scol - g0 : 4;
        if (nb == 4) st_b32(srow + g0, word);
        else st_partial(srow + g0, make_uint4(word, 0u, 0u, 0u), nb);
    }
}

// A warp owns a tile of RPS * U rows (RPS = 32 / TEAM rows side by side):
// lanes load the tile's slots once, then every lane issues the loads of its U
// rows before processing any of them.
template <int MODE, int TEAM>
__global__ void __launch_bounds__(IX_THREADS) indexer_quant_kernel(const IndexerArgs a) {
    constexpr int RPS = 32 / TEAM;
    constexpr int U = (32 / RPS) < 8 ? (32 / RPS) : 8;
    constexpr int TILE = RPS * U;
    const int lane = threadIdx.x & 31;
    const int tm = lane / TEAM;
    const int tl = lane % TEAM;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t ntiles = (a.T + TILE - 1) / TILE;
    const int nblocks = (a.nchunks + TEAM - 1) / TEAM;

    for (int64_t tile = gwarp; tile < ntiles; tile += nwarps) {
        const int64_t row0 = tile * TILE;
        const int rows = (int)(a.T - row0 < TILE ? a.T - row0 : TILE);
        int64_t my_slot = -1;
        if (lane < rows) {
            my_slot = load_slot(a.slots, a.slots_i64, row0 + lane);
            if (my_slot != -1 && !slot_ok(my_slot, a.cache.num_slots)) {
                raise_fault(FAULT_SLOT_RANGE);
                my_slot = -1;
            }
        }
        int64_t sl[U];
        bool live[U];
        const uint16_t* xrow[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = u * RPS + tm;
            const bool act = r < rows;
            sl[u] = __shfl_sync(FULL_MASK, my_slot, act ? r : 0);
            live[u] = act && sl[u] >= 0;
            xrow[u] = a.x + (row0 + (act ? r : 0)) * a.x_row_stride;
        }
        if (MODE == 1) {
            // fp8: one group per row -> row maximum, then quantise
            uint32_t m[U];
#pragma unroll
            for (int u = 0; u < U; ++u) m[u] = 0u;
            for (int cb = 0; cb < nblocks; ++cb) {
                const int c = cb * TEAM + tl;
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (live[u] && c < a.nchunks) m[u] = max(m[u], absmax_bits8(ix_load_chunk(a, xrow[u], c)));
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
#pragma unroll
                for (int k = TEAM / 2; k >= 1; k >>= 1) m[u] = max(m[u], __shfl_xor_sync(FULL_MASK, m[u], k));
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!live[u]) continue;
                const float scale = div_by_fmax(ix_amax(a, m[u]), a.e5m2 ? 57344.0f : 448.0f);
                uint8_t* crow = slot_row(a.cache, sl[u]);
                for (int cb = 0; cb < nblocks; ++cb) {
                    const int c = cb * TEAM + tl;
                    if (c >= a.nchunks) continue;
                    float f[8], q[8];
                    ix_widen(a, ix_load_chunk(a, xrow[u], c), f);
                    uint2 codes = make_uint2(0u, 0u);
                    if (scale != 0.0f) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(f[i], scale);
                        codes = ix_fp8x8(a, q);
                    }
                    const int nvalid = a.d - 8 * c;
                    if (nvalid >= 8) st_b64(crow + 8 * c, codes);
                    else st_partial(crow + 8 * c, make_uint4(codes.x, codes.y, 0u, 0u), nvalid);
                }
                if (tl == 0) st_b32(slot_row(a.scale, sl[u]), __float_as_uint(scale));
            }
        } else {
            for (int cb = 0; cb < nblocks; ++cb) {
                const int c = cb * TEAM + tl;
                uint4 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    v[u] = (live[u] && c < a.nchunks) ? ix_load_chunk(a, xrow[u], c) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int u = 0; u < U; ++u)
                    ix_mx_chunk<MODE, TEAM>(a, v[u], live[u], live[u] ? slot_row(a.cache, sl[u]) : nullptr,
                                            live[u] ? slot_row(a.scale, sl[u]) : nullptr, c, tl);
            }
        }
    }
}

}  // namespace kvq
