// indexer_quant.cuh -- indexer_quant_cache kernel (indexer_quant_cache,
// 接口功能: mxfp8 / mxfp4 groups of 32 with an E8M0 scale, fp8 one group per
// row with a binary32 scale; 约束说明 for the cache / cache_scale rows).
//
// One lane owns one 32-value quantisation group: it reads the group's 64
// bytes (two 32-byte loads when the rows allow it), takes the group maximum on
// its own, and writes the group's codes (32 bytes FP8, 16 bytes FP4) and its
// scale byte.  A row of ceil(d/32) groups is a TEAM of TG lanes (the next power
// of two, at most 32, walking the groups in steps of TG when there are more),
// so a warp covers 32/TG rows side by side.  The fp8 mode's row maximum is a
// butterfly over the team.  Grid-stride over passes of 32/TG rows; the slot of
// the next pass is loaded while the current one is quantised.  Rows whose slot
// is -1 are never read.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

struct IndexerArgs {
    const uint16_t* x;
    int64_t x_row_stride;
    int64_t T;
    int32_t d;
    int32_t ngroups;      // ceil(d / 32)
    int32_t team_shift;   // log2(lanes per row)
    int32_t x_vec;        // 2: rows 32-byte aligned, 1: 16-byte aligned, 0: neither
    const void* slots;
    int32_t slots_i64;
    PagedRows cache;      // codes
    PagedRows scale;      // cache_scale rows
    int32_t code_vec32;   // every code row starts on a 32-byte boundary
};

constexpr int IX_THREADS = 256;

template <bool F16>
__device__ __forceinline__ float ix_lo(uint32_t w) { return F16 ? f16_lo(w) : bf16_lo(w); }
template <bool F16>
__device__ __forceinline__ float ix_hi(uint32_t w) { return F16 ? f16_hi(w) : bf16_hi(w); }
template <bool F16>
__device__ __forceinline__ float ix_amax(uint32_t m) {
    return F16 ? __half2float(__ushort_as_half((unsigned short)m)) : __uint_as_float(m << 16);
}

// The values [32g, 32g + 32) of a row (zero beyond d) as 16 words.
__device__ __forceinline__ void ix_load_group(const IndexerArgs& a, const uint16_t* xrow, int g, uint32_t (&w)[16]) {
    const int nvalid = a.d - 32 * g;
    if (nvalid >= 32 && a.x_vec) {
        ld_slice(xrow + 32 * g, a.x_vec, w);
        return;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t lo = 2 * i < nvalid ? (uint32_t)__ldcs(xrow + 32 * g + 2 * i) : 0u;
        const uint32_t hi = 2 * i + 1 < nvalid ? (uint32_t)__ldcs(xrow + 32 * g + 2 * i + 1) : 0u;
        w[i] = lo | (hi << 16);
    }
}

// FP8 codes of the 32 values of w, each multiplied (DIV false) or divided
// (DIV true) by s
template <bool F16, bool E5M2, bool DIV>
__device__ __forceinline__ void ix_fp8_codes(const uint32_t (&w)[16], float s, uint32_t (&c)[8]) {
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        float q[4] = {ix_lo<F16>(w[i]), ix_hi<F16>(w[i]), ix_lo<F16>(w[i + 1]), ix_hi<F16>(w[i + 1])};
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = DIV ? __fdiv_rn(q[k], s) : __fmul_rn(q[k], s);
        c[i / 2] = fp8x2<E5M2>(q[0], q[1]) | (fp8x2<E5M2>(q[2], q[3]) << 16);
    }
}

// fp8 mode: whether the row's codes may come from the two-step quotient
// (div_scale2 with r = RN(1/scale)) instead of IEEE division.  For a finite
// amax >= 2^-60, scale = RN(amax / FMAX) and r are normal; a value with
// |x| >= 2^-100 has a normal quotient and normal residuals, so the two-step
// form returns exactly the IEEE quotient (Markstein, IBM J. Res. Dev. 34(1),
// 1990); a smaller |x| has a quotient below 2^-23 in magnitude either way,
// whose code is the signed zero of x's sign either way.  kvq_selftest 8
// checks the codes of both paths against each other.
__device__ __forceinline__ bool ix_fp8_fast(float amax) {
    return amax >= 8.673617379884035e-19f && amax <= 3.4028234663852886e38f;   // [2^-60, FLT_MAX]
}

// FP8 codes of the 32 values of w divided by s through the two-step quotient
template <bool F16, bool E5M2>
__device__ __forceinline__ void ix_fp8_codes_q2(const uint32_t (&w)[16], float s, float r, uint32_t (&c)[8]) {
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        float q[4] = {ix_lo<F16>(w[i]), ix_hi<F16>(w[i]), ix_lo<F16>(w[i + 1]), ix_hi<F16>(w[i + 1])};
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = div_scale2(q[k], s, r);
        c[i / 2] = fp8x2<E5M2>(q[0], q[1]) | (fp8x2<E5M2>(q[2], q[3]) << 16);
    }
}

// The first nbytes (<= 32) of the 8 code words at p
__device__ __forceinline__ void ix_store_codes(uint8_t* p, const uint32_t (&c)[8], int nbytes, bool vec32) {
    if (nbytes >= 32) {
        st_32B(p, c, vec32);
        return;
    }
#pragma unroll
    for (int k = 0; k < 32; ++k)
        if (k < nbytes) p[k] = (uint8_t)(c[k >> 2] >> (8 * (k & 3)));
}

template <int MODE, bool F16, bool E5M2>
__global__ void __launch_bounds__(IX_THREADS) indexer_quant_kernel(const IndexerArgs a) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int ts = a.team_shift;
    const int TG = 1 << ts;
    const int tm = lane >> ts;                 // row within the pass
    const int gl = lane & (TG - 1);            // first group of this lane
    const int rpp = 32 >> ts;                  // rows per pass
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t npass = (a.T + rpp - 1) / rpp;
    const bool v32 = a.code_vec32 != 0;
    constexpr float FMAX = MODE == 3 ? 6.0f : (E5M2 ? 57344.0f : 448.0f);

    auto slot_of = [&](int64_t pass) -> int64_t {
        const int64_t row = pass * rpp + tm;
        if (pass >= npass || row >= a.T) return -1;
        return load_slot(a.slots, a.slots_i64, row);
    };
    int64_t s_next = slot_of(gwarp);
    for (int64_t pass = gwarp; pass < npass; pass += nwarps) {
        const int64_t row = pass * rpp + tm;
        const int64_t s = s_next;
        s_next = slot_of(pass + nwarps);
        bool live = false;
        if (s != -1) {
            if (slot_ok(s, a.cache.num_slots)) live = true;
            else if (gl == 0) raise_fault(FAULT_SLOT_RANGE);
        }
        const uint16_t* xrow = a.x + (live ? row : 0) * a.x_row_stride;
        uint8_t* crow = live ? slot_row(a.cache, s) : nullptr;
        uint8_t* srow = live ? slot_row(a.scale, s) : nullptr;

        if (MODE == 1) {
            // fp8: one binary32 scale per row = row maximum / FP8_MAX
            uint32_t w[16];
            uint32_t m = 0u;
            const bool keep = a.ngroups <= TG;     // each lane holds at most one group
            for (int g = gl; g < a.ngroups; g += TG) {
                if (!live) break;
                ix_load_group(a, xrow, g, w);
                m = max(m, absmax_words<16>(w, 0));
            }
            for (int k = TG >> 1; k >= 1; k >>= 1) m = max(m, __shfl_xor_sync(FULL_MASK, m, k));
            if (!live) continue;
            const float amax = ix_amax<F16>(m);
            const float scale = div_by_fmax(amax, FMAX);
            const bool fast = ix_fp8_fast(amax);
            const float r = fast ? __frcp_rn(scale) : 0.0f;
            for (int g = gl; g < a.ngroups; g += TG) {
                if (!keep) ix_load_group(a, xrow, g, w);
                uint32_t c[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                if (fast) ix_fp8_codes_q2<F16, E5M2>(w, scale, r, c);
                else if (scale != 0.0f) ix_fp8_codes<F16, E5M2, true>(w, scale, c);
                ix_store_codes(crow + 32 * g, c, a.d - 32 * g, v32);
            }
            if (gl == 0) st_b32(srow, __float_as_uint(scale));
            continue;
        }
        if (!live) continue;
        for (int g = gl; g < a.ngroups; g += TG) {
            uint32_t w[16];
            ix_load_group(a, xrow, g, w);
            // E8M0 scale: group maximum / FMAX rounded up to a power of two
            const uint32_t b = e8m0_ceil(div_by_fmax(ix_amax<F16>(absmax_words<16>(w, 0)), FMAX));
            const float mul = e8m0_reciprocal(b);
            const int nvalid = a.d - 32 * g;
            if (MODE == 0) {
                uint32_t c[8];
                ix_fp8_codes<F16, E5M2, false>(w, mul, c);
                ix_store_codes(crow + 32 * g, c, nvalid, v32);
            } else {
                uint32_t c[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
                for (int i = 0; i < 16; i += 4) {
                    float q[8];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        q[2 * k] = __fmul_rn(ix_lo<F16>(w[i + k]), mul);
                        q[2 * k + 1] = __fmul_rn(ix_hi<F16>(w[i + k]), mul);
                    }
                    c[i / 4] = e2m1x8(q);
                }
                if (nvalid >= 32) st_b128(crow + 16 * g, make_uint4(c[0], c[1], c[2], c[3]));
                else ix_store_codes(crow + 16 * g, c, (nvalid + 1) / 2, false);
            }
            st_b8(srow + g, b);
        }
    }
}

}  // namespace kvq
