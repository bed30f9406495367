// rmsnorm_rope.cuh -- kv_rmsnorm_rope_cache kernel (aclnnKvRmsNormRopeCache,
// 计算公式 (1) interleaveRope and (2) rmsNorm; 约束说明 for index modes and
// cache dtype scenarios).
//
// One warp per token.  The sum of squares follows the library's fixed order:
// value i of the RMSNorm segment belongs to 8-value chunk i/8, chunk c to lane
// c % 32; each lane adds x*x of its values in index order, then the lanes
// combine by the butterfly p += p[lane ^ k], k = 16, 8, 4, 2, 1.  Aligned rows
// are read as 16-byte chunks kept in registers for the normalisation and
// written back as 8- or 16-byte chunks; other rows element by element (the
// row read twice, the second time from L1).  The rope segment is handled one
// interleaved pair per lane.  gamma, cos and sin are small and stay in L1/L2
// across tokens.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

enum CacheDt : int32_t { CDT_BF16 = 0, CDT_F16 = 1, CDT_E4M3 = 2, CDT_E5M2 = 3, CDT_I8 = 4 };

struct CacheOut {
    PagedRows rows;
    int32_t dt;             // CacheDt
    const float* scale;     // null, 1 value, or one per channel
    int32_t scale_n;
    const float* offset;    // int8 only: null, 1 value, or one per channel
    int32_t offset_n;
};

struct RmsRopeArgs {
    const uint16_t* kv;     // [B, 1, S, D] contiguous
    int32_t kv_f16;
    int64_t B, S;
    int32_t D, Dv, Dk;
    const uint16_t* gamma;  // [Dv]
    const uint16_t* cos;    // [B*S, Dk]
    const uint16_t* sin;
    const void* index;
    int32_t index_i64;
    int32_t cache_mode;     // 0 Norm, 1 PA, 2 PA_BNSD, 3 PA_BLK_BNSD
    CacheOut k;             // Dk values per row
    CacheOut ckv;           // Dv values per row
    float eps;
    int32_t ckv_stage;      // int8 ckv: scales, offsets and reciprocals staged in shared memory ([3][Dv])
    float inv_dv;           // 1 / Dv when Dv is a power of two (exact), else 0
};

constexpr int RR_THREADS = 128;

__device__ __forceinline__ float half_bits(uint32_t h, int f16) {
    return f16 ? __half2float(__ushort_as_half((unsigned short)h)) : __uint_as_float(h << 16);
}

__device__ __forceinline__ float half_at(const uint16_t* p, int64_t i, int f16) {
    return half_bits(p[i], f16);
}

// Store y as element j of a cache row (unquantised: rounded to the dtype;
// quantised: fp(y / scale) or int8(rint(y / scale + offset))).
__device__ __forceinline__ void store_elem(const CacheOut& c, uint8_t* row, int j, float y) {
    switch (c.dt) {
        case CDT_BF16: st_b16(row + 2 * j, to_bf16_bits(y)); break;
        case CDT_F16: st_b16(row + 2 * j, to_f16_bits(y)); break;
        case CDT_E4M3:
        case CDT_E5M2: {
            const float s = c.scale[c.scale_n == 1 ? 0 : j];
            const float q = __fdiv_rn(y, s);
            row[j] = (uint8_t)(c.dt == CDT_E4M3 ? e4m3x2(q, 0.0f) : e5m2x2(q, 0.0f));
            break;
        }
        case CDT_I8: {
            const float s = c.scale[c.scale_n == 1 ? 0 : j];
            float q = __fdiv_rn(y, s);
            if (c.offset) q = __fadd_rn(q, c.offset[c.offset_n == 1 ? 0 : j]);
            row[j] = (uint8_t)int8_rne_sat(q);
            break;
        }
        default: break;
    }
}

// Token t's batch b and position s (needed by the Norm and PA_BLK_BNSD modes
// only; 0 otherwise) and the position of its entry in the index tensor.
__device__ __forceinline__ int64_t rr_index_pos(const RmsRopeArgs& a, int64_t t, int64_t& b, int64_t& s) {
    b = 0;
    s = 0;
    if (a.cache_mode != 0 && a.cache_mode != 3) return t;  // PA, PA_BNSD: one entry per token
    b = t / a.S;
    s = t - b * a.S;
    if (a.cache_mode == 0) return t;
    const int64_t bs = a.k.rows.block_size;
    return b * ((a.S + bs - 1) / bs) + s / bs;               // PA_BLK_BNSD: one entry per block of tokens
}

// Destination slot of token (b, s) from its index entry v: >= 0 a slot, -1
// skip, -2 out of range.
__device__ __forceinline__ int64_t rr_resolve(const RmsRopeArgs& a, int64_t b, int64_t s, int64_t v) {
    const int64_t bs = a.k.rows.block_size;
    if (v == -1) return -1;
    if (a.cache_mode == 0) {                       // Norm: [B, S] positions, one block per batch
        if (v < 0 || v >= bs || b * bs >= a.k.rows.num_slots) return -2;
        return b * bs + v;
    }
    if (v < 0 || v >= a.k.rows.num_slots) return -2;
    if (a.cache_mode == 3) return (v / bs) * bs + s % bs;
    return v;                                      // PA, PA_BNSD
}

// A per-tensor ckv scale s in [2^-40, 2^40] and r = RN(1/s): the FP8 codes of
// y / s come from the two-step quotient (div2_x2) for chunks with every
// |y| <= 2^60.  It is exact for |y| >= 2^-103 (the residual is then a
// multiple of 2^-149, so the fused operations form it exactly, and the
// quotient stays normal); a smaller |y| has |y / s| < 2^-63, whose code is
// the zero of y's sign either way.
// A per-tensor ckv scale that is a normal power of two, s = 2^e: r = 1/s is
// exact, and RN(y r) and RN(y / s) are the same single rounding of the same
// real number (subnormal results included), so the codes come from one
// multiply (pow2).
struct CkvDiv {
    float s, r;
    bool fast;
    bool pow2;
};

// The ckv cache's dtype class, a template parameter of the register kernels
// so that each instantiation carries only its own store path: 0 bf16 / f16,
// 1 FP8 (E4M3 / E5M2), 2 int8.
__host__ __device__ inline int ckv_class(int32_t dt) {
    return dt == CDT_I8 ? 2 : ((dt == CDT_E4M3 || dt == CDT_E5M2) ? 1 : 0);
}

// y[0..7] = chunk c of the RMSNorm segment normalised and scaled, stored as
// the ckv cache's dtype (8 values at row element 8c); CK: ckv_class(c.dt)
template <int CK>
__device__ __forceinline__ void rr_store_chunk(const CacheOut& c, uint8_t* row, int ch, const float (&y)[8],
                                               const CkvDiv& dv, const float* stg, int Dv) {
    const int j0 = 8 * ch;
    switch (CK == 0 ? CDT_BF16 : (CK == 1 ? CDT_E4M3 : CDT_I8)) {
        case CDT_BF16: {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t lo = c.dt == CDT_BF16 ? to_bf16_bits(y[2 * k]) : to_f16_bits(y[2 * k]);
                const uint32_t hi = c.dt == CDT_BF16 ? to_bf16_bits(y[2 * k + 1]) : to_f16_bits(y[2 * k + 1]);
                w[k] = lo | (hi << 16);
            }
            st_b128(row + 2 * j0, make_uint4(w[0], w[1], w[2], w[3]));
            break;
        }
        case CDT_E4M3: {
            float q[8];
            if (dv.pow2) {
#pragma unroll
                for (int k = 0; k < 8; k += 2) mul_x2(y[k], y[k + 1], dv.r, dv.r, q[k], q[k + 1]);
                st_b64(row + j0, c.dt == CDT_E4M3 ? fp8x8<false>(q) : fp8x8<true>(q));
                break;
            }
            float ym = 0.0f;
#pragma unroll
            for (int k = 0; k < 8; ++k) ym = fmaxf(ym, fabsf(y[k]));
            if (dv.fast && ym <= 1.152921504606846976e18f) {            // 2^60
#pragma unroll
                for (int k = 0; k < 8; k += 2) div2_x2(y[k], y[k + 1], dv.s, dv.r, q[k], q[k + 1]);
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) q[k] = __fdiv_rn(y[k], c.scale[c.scale_n == 1 ? 0 : j0 + k]);
            }
            st_b64(row + j0, c.dt == CDT_E4M3 ? fp8x8<false>(q) : fp8x8<true>(q));
            break;
        }
        case CDT_I8: {
            if (stg) {
                // the staged per-channel scale, offset and RN(1/scale): int8x4_quant
                uint32_t w[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float4 sv = *reinterpret_cast<const float4*>(stg + j0 + 4 * h);
                    const float4 fv = *reinterpret_cast<const float4*>(stg + Dv + j0 + 4 * h);
                    const float4 rv = *reinterpret_cast<const float4*>(stg + 2 * Dv + j0 + 4 * h);
                    const float o4[4] = {y[4 * h], y[4 * h + 1], y[4 * h + 2], y[4 * h + 3]};
                    const float s4[4] = {sv.x, sv.y, sv.z, sv.w}, f4[4] = {fv.x, fv.y, fv.z, fv.w};
                    const float r4[4] = {rv.x, rv.y, rv.z, rv.w};
                    w[h] = int8x4_quant(o4, s4, f4, r4);
                }
                st_b64(row + j0, make_uint2(w[0], w[1]));
                break;
            }
            uint32_t w[2] = {0u, 0u};
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                float q = __fdiv_rn(y[k], c.scale[c.scale_n == 1 ? 0 : j0 + k]);
                if (c.offset) q = __fadd_rn(q, c.offset[c.offset_n == 1 ? 0 : j0 + k]);
                w[k >> 2] |= ((uint32_t)int8_rne_sat(q) & 0xffu) << (8 * (k & 3));
            }
            st_b64(row + j0, make_uint2(w[0], w[1]));
            break;
        }
        default: break;
    }
}

// NCH == 0: element-wise loads (any alignment, any Dv).  NCH > 0: 16-byte
// rows (kv, gamma 16-byte aligned, D and Dv multiples of 8) with at most
// 32 * NCH chunks: each lane keeps its chunks c = lane, lane + 32, ... in
// registers between the sum of squares and the normalisation.
// Eight CTAs of four warps per SM (at most 64 registers): the kernel is bound
// by latency and the two IEEE divisions per value, and runs faster with more
// warps resident (79 us at 8 CTAs per SM vs 93 us at 5 for 65,536 tokens).
template <int NCH, int CK = 0>
__global__ void __launch_bounds__(RR_THREADS, 8) rmsnorm_rope_kernel(const RmsRopeArgs a) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t ntok = a.B * a.S;
    const int nch = (a.Dv + 7) / 8;
    const int h = a.Dk / 2;

    // register kernel: the next token's RMSNorm chunks are loaded while the
    // current token is normalised (a token's row is read whether or not it is
    // skipped)
    uint4 xn[NCH > 0 ? NCH : 1];
    auto load_chunks = [&](int64_t t, uint4 (&v)[NCH > 0 ? NCH : 1]) {
#pragma unroll
        for (int m = 0; m < NCH; ++m) {
            const int c = lane + 32 * m;
            v[m] = (t < ntok && c < nch) ? __ldg(reinterpret_cast<const uint4*>(a.kv + t * a.D) + c)
                                         : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    // the next token's index entry (and, with at most 32 RoPE pairs, each
    // lane's RoPE inputs) are loaded while the current token is processed
    const bool rope_pf = NCH > 0 && h <= 32;
    int64_t v_next = -1, b_next = 0, s_next = 0;
    uint32_t zn = 0u, cn = 0u, sn = 0u;
    auto prefetch = [&](int64_t t) {
        if (t >= ntok) return;
        v_next = load_slot(a.index, a.index_i64, rr_index_pos(a, t, b_next, s_next));
        if (rope_pf && lane < h) {
            const uint16_t* z = a.kv + t * a.D + a.Dv;
            zn = (uint32_t)z[2 * lane] | ((uint32_t)z[2 * lane + 1] << 16);
            cn = (uint32_t)a.cos[t * a.Dk + lane] | ((uint32_t)a.cos[t * a.Dk + h + lane] << 16);
            sn = (uint32_t)a.sin[t * a.Dk + lane] | ((uint32_t)a.sin[t * a.Dk + h + lane] << 16);
        }
    };
    // int8 ckv: per-channel scale, offset (0 when absent) and the reciprocal
    // of int8x4_quant, staged once per CTA
    extern __shared__ __align__(16) float rr_stage[];
    const float* stg = nullptr;
    if (NCH > 0 && CK == 2 && a.ckv_stage) {
        for (int i = threadIdx.x; i < a.Dv; i += blockDim.x) {
            const float sc = a.ckv.scale[a.ckv.scale_n == 1 ? 0 : i];
            const float of = a.ckv.offset ? a.ckv.offset[a.ckv.offset_n == 1 ? 0 : i] : 0.0f;
            rr_stage[i] = sc;
            rr_stage[a.Dv + i] = of;
            rr_stage[2 * a.Dv + i] = int8_quant_rcp(sc, of);
        }
        __syncthreads();
        stg = rr_stage;
    }
    CkvDiv dv{0.0f, 0.0f, false, false};
    if (NCH > 0 && CK == 1 && a.ckv.scale_n == 1) {
        dv.s = a.ckv.scale[0];
        const uint32_t sb = __float_as_uint(dv.s);
        dv.pow2 = (sb & 0x807fffffu) == 0u && (sb >> 23) >= 1u && (sb >> 23) <= 254u;   // +2^e, normal
        dv.fast = dv.s >= 9.094947017729282e-13f && dv.s <= 1.099511627776e12f;        // [2^-40, 2^40]
        dv.r = (dv.fast || dv.pow2) ? __frcp_rn(dv.s) : 0.0f;
    }
    if (NCH > 0) load_chunks(gwarp, xn);
    prefetch(gwarp);
    for (int64_t t = gwarp; t < ntok; t += nwarps) {
        uint4 xv[NCH > 0 ? NCH : 1];
        if (NCH > 0) {
#pragma unroll
            for (int m = 0; m < NCH; ++m) xv[m] = xn[m];
            load_chunks(t + nwarps, xn);
        }
        const int64_t slot = rr_resolve(a, b_next, s_next, v_next);     // warp-uniform
        const uint32_t zr = zn, cr = cn, sr = sn;
        prefetch(t + nwarps);
        if (slot == -2) {
            if (lane == 0) raise_fault(FAULT_SLOT_RANGE);
            continue;
        }
        if (slot < 0) continue;
        const uint16_t* x = a.kv + t * a.D;
        uint8_t* crow = slot_row(a.ckv.rows, slot);

        if (NCH > 0) {
            // RMSNorm: sum of squares in the fixed lane order, chunks from registers;
            // also the smallest exponent field of the lane's values (per 16-bit
            // half, on the raw bits): every value then has |x| >= 2^(e - bias),
            // and a zero or subnormal value gives e = 0
            // (fused square-accumulate, sq_acc8: exact for f16, and for bf16
            // lanes whose values all have |x| >= 2^-67; a lane with a smaller
            // or zero value sums again with the square rounded first)
            float acc = 0.0f;
            const uint32_t emask = a.kv_f16 ? 0x7c007c00u : 0x7f807f80u;
            uint32_t emin2 = emask;
#pragma unroll
            for (int m = 0; m < NCH; ++m) {
                if (lane + 32 * m >= nch) break;
                acc = a.kv_f16 ? sq_acc8<true>(xv[m], acc) : sq_acc8<false>(xv[m], acc);
                emin2 = __vminu2(emin2, __vminu2(xv[m].x & emask, xv[m].y & emask));
                emin2 = __vminu2(emin2, __vminu2(xv[m].z & emask, xv[m].w & emask));
            }
            const uint32_t emin = min(emin2 & 0xffffu, emin2 >> 16);     // 2^(e - bias) as 16-bit float bits
            if (!a.kv_f16 && emin < 0x1e00u) {                           // 2^-67 as bf16
                acc = 0.0f;
#pragma unroll
                for (int m = 0; m < NCH; ++m) {
                    if (lane + 32 * m >= nch) break;
                    float f[8];
                    widen8<false>(xv[m], f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc = __fadd_rn(acc, __fmul_rn(f[i], f[i]));
                }
            }
#pragma unroll
            for (int k = 16; k >= 1; k >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(FULL_MASK, acc, k));
            const float mean = a.inv_dv != 0.0f ? __fmul_rn(acc, a.inv_dv) : __fdiv_rn(acc, (float)a.Dv);
            const float rms = __fsqrt_rn(__fadd_rn(mean, a.eps));
            // x / rms by one correction step (div1_x2_nz): RN(x / rms) when rms
            // is in [2^-60, 2^50] and, per lane, every |x| is nonzero and at
            // least max(RN(rms 2^-125), 2^-103) -- the reciprocal and the
            // quotient are then normal and the residual x - q rms a multiple of
            // 2^-149, formed exactly by the fused operation (kvq_selftest 9 and
            // 10 check the domain; a subnormal quotient can be an exact
            // rounding tie, which the short form may break the wrong way, hence
            // the first bound), and a nonzero numerator's quotient keeps its
            // sign without a fix.  The lane's smallest power of two
            // 2^(e - bias) stands for its values; a lane with a zero or a
            // smaller value divides with IEEE division.
            const float uthr = fmaxf(__fmul_rn(rms, 2.350988701644575e-38f), 9.860761315262648e-32f);
            const bool ufast = rms >= 8.673617379884035e-19f && rms <= 1.125899906842624e15f &&
                               half_bits(emin, a.kv_f16) >= uthr;
            const float rr1 = ufast ? __frcp_rn(rms) : 0.0f;
#pragma unroll
            for (int m = 0; m < NCH; ++m) {
                const int c = lane + 32 * m;
                if (c >= nch) break;
                float f[8], g[8], y[8];
                const uint4 gv = __ldg(reinterpret_cast<const uint4*>(a.gamma) + c);
                if (a.kv_f16) {
                    widen8<true>(xv[m], f);
                    widen8<true>(gv, g);
                } else {
                    widen8<false>(xv[m], f);
                    widen8<false>(gv, g);
                }
                if (ufast) {
#pragma unroll
                    for (int i = 0; i < 8; i += 2) div1_x2_nz(f[i], f[i + 1], rms, rr1, y[i], y[i + 1]);
#pragma unroll
                    for (int i = 0; i < 8; i += 2) mul_x2(y[i], y[i + 1], g[i], g[i + 1], y[i], y[i + 1]);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) y[i] = __fmul_rn(__fdiv_rn(f[i], rms), g[i]);
                }
                rr_store_chunk<CK>(a.ckv, crow, c, y, dv, stg, a.Dv);
            }
        } else {
            // RMSNorm: sum of squares in the fixed lane order
            float acc = 0.0f;
            for (int c = lane; c < nch; c += 32) {
                for (int i = 8 * c; i < 8 * c + 8 && i < a.Dv; ++i) {
                    const float v = half_at(x, i, a.kv_f16);
                    acc = __fadd_rn(acc, __fmul_rn(v, v));
                }
            }
#pragma unroll
            for (int k = 16; k >= 1; k >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(FULL_MASK, acc, k));
            const float mean = __fdiv_rn(acc, (float)a.Dv);
            const float rms = __fsqrt_rn(__fadd_rn(mean, a.eps));
            for (int c = lane; c < nch; c += 32) {
                for (int i = 8 * c; i < 8 * c + 8 && i < a.Dv; ++i) {
                    const float v = half_at(x, i, a.kv_f16);
                    const float y = __fmul_rn(__fdiv_rn(v, rms), half_at(a.gamma, i, a.kv_f16));
                    store_elem(a.ckv, crow, i, y);
                }
            }
        }

        uint8_t* krow = slot_row(a.k.rows, slot);
        if (rope_pf) {
            // interleaved RoPE on the prefetched pair of this lane
            if (lane < h) {
                const float z0 = half_bits(zr & 0xffffu, a.kv_f16), z1 = half_bits(zr >> 16, a.kv_f16);
                const float c0 = half_bits(cr & 0xffffu, a.kv_f16), c1 = half_bits(cr >> 16, a.kv_f16);
                const float s0 = half_bits(sr & 0xffffu, a.kv_f16), s1 = half_bits(sr >> 16, a.kv_f16);
                store_elem(a.k, krow, lane, __fadd_rn(__fmul_rn(z0, c0), __fmul_rn(-z1, s0)));
                store_elem(a.k, krow, h + lane, __fadd_rn(__fmul_rn(z1, c1), __fmul_rn(z0, s1)));
            }
            continue;
        }
        // interleaved RoPE: y_j = z_2j c_j - z_2j+1 s_j, y_h+j = z_2j+1 c_h+j + z_2j s_h+j
        const uint16_t* z = x + a.Dv;
        const uint16_t* cs = a.cos + t * a.Dk;
        const uint16_t* sn = a.sin + t * a.Dk;
        for (int j = lane; j < h; j += 32) {
            const float z0 = half_at(z, 2 * j, a.kv_f16), z1 = half_at(z, 2 * j + 1, a.kv_f16);
            const float c0 = half_at(cs, j, a.kv_f16), c1 = half_at(cs, h + j, a.kv_f16);
            const float s0 = half_at(sn, j, a.kv_f16), s1 = half_at(sn, h + j, a.kv_f16);
            const float y0 = __fadd_rn(__fmul_rn(z0, c0), __fmul_rn(-z1, s0));
            const float y1 = __fadd_rn(__fmul_rn(z1, c1), __fmul_rn(z0, s1));
            store_elem(a.k, krow, j, y0);
            store_elem(a.k, krow, h + j, y1);
        }
    }
}

// ---------------------------------------------------------------------------
// The lean kernel: rows of the common shape -- Dv = 256 NCH RMSNorm values
// (lane l owns the 16-byte chunks l + 32 m), Dk = 64 RoPE values (one
// interleaved pair per lane), one index entry per token (PA, PA_BNSD), fewer
// than 2^31 tokens and slots, cache rows aligned for whole-chunk stores.  It
// computes exactly what rmsnorm_rope_kernel computes, with less work per
// token: 32-bit token and slot arithmetic, the dtypes as template parameters
// (CK: 0 bf16 / f16 ckv, 1 E4M3, 2 int8, 3 E5M2; KF16: f16 kv, gamma, cos,
// sin), the sum of squares by fused 16-bit multiply-adds (sq_acc8), x / rms
// by one correction step (div1_x2_nz), and gamma staged per CTA as binary32.
//
// For an E4M3 / E5M2 ckv cache with a per-tensor scale s = 2^-k, 0 <= k <= 109,
// the staged gamma is g r with r = 2^k (exact when every finite g keeps a
// finite g r), and y r = RN(q g) r becomes RN(q (g r)): in the normal range a
// power-of-two factor commutes with rounding, an overflow overflows in both
// forms, and where RN(q g) is subnormal both results are at most 2^-17 in
// magnitude, which both formats encode as the zero of the same sign.
// ---------------------------------------------------------------------------
// The staged gamma (g, or g r when the FP8 scale folds in) and, for an int8
// ckv cache, its per-channel scale, offset and RN(1/scale) ([3][DV] at stg),
// written by the CTA's threads; returns whether the scale folded in.  dv
// receives the per-tensor FP8 scale forms.  Every thread of the CTA calls it.
template <int NCH, int CK, bool KF16>
__device__ __forceinline__ bool rr_lean_stage(const RmsRopeArgs& a, float* gs, float* stg, CkvDiv& dv) {
    constexpr int DV = 256 * NCH;
    constexpr bool FP8 = CK == 1 || CK == 3;
    dv = CkvDiv{0.0f, 0.0f, false, false};
    bool pow2 = false;
    if (FP8 && a.ckv.scale_n == 1) {
        dv.s = a.ckv.scale[0];
        const uint32_t sb = __float_as_uint(dv.s);
        dv.pow2 = (sb & 0x807fffffu) == 0u && (sb >> 23) >= 1u && (sb >> 23) <= 254u;
        dv.fast = dv.s >= 9.094947017729282e-13f && dv.s <= 1.099511627776e12f;
        dv.r = (dv.fast || dv.pow2) ? __frcp_rn(dv.s) : 0.0f;
        pow2 = dv.pow2 && (sb >> 23) >= 18u && (sb >> 23) <= 127u;   // s = 2^-k, 0 <= k <= 109
    }
    int ok = 1;
    for (int i = threadIdx.x; i < DV; i += blockDim.x) {
        const float g = half_bits(a.gamma[i], KF16);
        gs[i] = g;
        if (pow2 && fabsf(g) <= 3.4028234663852886e38f && !(fabsf(__fmul_rn(g, dv.r)) <= 3.4028234663852886e38f))
            ok = 0;
        if (CK == 2) {
            const float sc = a.ckv.scale[a.ckv.scale_n == 1 ? 0 : i];
            const float of = a.ckv.offset ? a.ckv.offset[a.ckv.offset_n == 1 ? 0 : i] : 0.0f;
            stg[i] = sc;
            stg[DV + i] = of;
            stg[2 * DV + i] = int8_quant_rcp(sc, of);
        }
    }
    const bool fold = __syncthreads_and(ok) && pow2;
    if (fold) {
        for (int i = threadIdx.x; i < DV; i += blockDim.x) gs[i] = __fmul_rn(gs[i], dv.r);
        __syncthreads();
    }
    return fold;
}

// One token of the lean kernels, computed by one warp: RMSNorm of this lane's
// chunks xv[m] (values 8 (lane + 32 m) .. + 7) into the ckv cache row and
// RoPE of its pair j = lane (zr: values Dv + 2j, Dv + 2j + 1; cr, sr: cos and
// sin at j and 32 + j) into the k cache row, both rows of cache slot `slot`.
template <int NCH, int CK, bool KF16>
__device__ __forceinline__ void rr_lean_token(const RmsRopeArgs& a, const uint4 (&xv)[NCH], uint32_t zr, uint32_t cr,
                                              uint32_t sr, uint32_t slot, const float* gs, const float* stg,
                                              const CkvDiv& dv, bool fold, int lane) {
    constexpr int DV = 256 * NCH;
    constexpr bool FP8 = CK == 1 || CK == 3;
    const uint32_t bsz = (uint32_t)a.k.rows.block_size;
    const int sh = a.k.rows.bs_shift;
    const uint32_t blk = sh >= 0 ? slot >> sh : slot / bsz;
    const uint32_t row = slot - blk * bsz;
    uint8_t* crow = a.ckv.rows.base + (uint64_t)blk * (uint32_t)a.ckv.rows.block_stride +
                    row * (uint32_t)a.ckv.rows.row_bytes;
    uint8_t* krow = a.k.rows.base + (uint64_t)blk * (uint32_t)a.k.rows.block_stride +
                    row * (uint32_t)a.k.rows.row_bytes;

    // RMSNorm: the sum of squares in the fixed lane order and the lane's
    // smallest |x| (as 16-bit float bits)
    float acc = 0.0f;
    uint32_t mn = 0x7fff7fffu;
#pragma unroll
    for (int m = 0; m < NCH; ++m) {
        acc = sq_acc8<KF16>(xv[m], acc);
        mn = absmin_x2<KF16>(mn, absmin_x2<KF16>(absmin_x2<KF16>(xv[m].x, xv[m].y),
                                                 absmin_x2<KF16>(xv[m].z, xv[m].w)));
    }
    mn &= 0x7fff7fffu;
    const uint32_t emin = min(mn & 0xffffu, mn >> 16);
    if (!KF16 && emin < 0x1e00u) {                    // a bf16 value below 2^-67, or zero
        acc = 0.0f;
#pragma unroll
        for (int m = 0; m < NCH; ++m) {
            float f[8];
            widen8<false>(xv[m], f);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc = __fadd_rn(acc, __fmul_rn(f[i], f[i]));
        }
    }
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(FULL_MASK, acc, k));
    const float mean = __fmul_rn(acc, 1.0f / (float)DV);              // exact: DV is a power of two
    const float rms = __fsqrt_rn(__fadd_rn(mean, a.eps));
    // the guard of the one-step quotient (as in rmsnorm_rope_kernel)
    const float uthr = fmaxf(__fmul_rn(rms, 2.350988701644575e-38f), 9.860761315262648e-32f);
    const bool ufast = rms >= 8.673617379884035e-19f && rms <= 1.125899906842624e15f &&
                       half_bits(emin, KF16) >= uthr;
    const float rr1 = ufast ? __frcp_rn(rms) : 0.0f;
#pragma unroll
    for (int m = 0; m < NCH; ++m) {
        const int c = lane + 32 * m;
        float f[8], y[8];
        widen8<KF16>(xv[m], f);
        if (ufast) {
#pragma unroll
            for (int i = 0; i < 8; i += 2) div1_x2_nz(f[i], f[i + 1], rms, rr1, y[i], y[i + 1]);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = __fdiv_rn(f[i], rms);
        }
        const float4 g0 = *reinterpret_cast<const float4*>(gs + 8 * c);
        const float4 g1 = *reinterpret_cast<const float4*>(gs + 8 * c + 4);
        mul_x2(y[0], y[1], g0.x, g0.y, y[0], y[1]);
        mul_x2(y[2], y[3], g0.z, g0.w, y[2], y[3]);
        mul_x2(y[4], y[5], g1.x, g1.y, y[4], y[5]);
        mul_x2(y[6], y[7], g1.z, g1.w, y[6], y[7]);
        if (CK == 0) {
            uint4 w;
            if (a.ckv.dt == CDT_BF16)
                w = make_uint4(half2_bits<false>(y[0], y[1]), half2_bits<false>(y[2], y[3]),
                               half2_bits<false>(y[4], y[5]), half2_bits<false>(y[6], y[7]));
            else
                w = make_uint4(half2_bits<true>(y[0], y[1]), half2_bits<true>(y[2], y[3]),
                               half2_bits<true>(y[4], y[5]), half2_bits<true>(y[6], y[7]));
            *reinterpret_cast<uint4*>(crow + 16 * c) = w;
        } else if (FP8) {
            if (fold) *reinterpret_cast<uint2*>(crow + 8 * c) = fp8x8_packed<CK == 3>(y);
            else rr_store_chunk<1>(a.ckv, crow, c, y, dv, nullptr, DV);
        } else {
            rr_store_chunk<2>(a.ckv, crow, c, y, dv, stg, DV);
        }
    }

    // interleaved RoPE on this lane's pair j = lane:
    // y_j = z_2j c_j - z_2j+1 s_j, y_32+j = z_2j+1 c_32+j + z_2j s_32+j
    // (scalar products and sums: -fmad=false keeps them separately rounded,
    // where a packed product followed by a packed add may be fused)
    const float z0 = half_bits(zr & 0xffffu, KF16), z1 = half_bits(zr >> 16, KF16);
    const float c0 = half_bits(cr & 0xffffu, KF16), c1 = half_bits(cr >> 16, KF16);
    const float s0 = half_bits(sr & 0xffffu, KF16), s1 = half_bits(sr >> 16, KF16);
    const float y0 = __fadd_rn(__fmul_rn(z0, c0), __fmul_rn(-z1, s0));
    const float y1 = __fadd_rn(__fmul_rn(z1, c1), __fmul_rn(z0, s1));
    if (a.k.dt == CDT_BF16 || a.k.dt == CDT_F16) {
        const uint32_t w = a.k.dt == CDT_BF16 ? half2_bits<false>(y0, y1) : half2_bits<true>(y0, y1);
        *reinterpret_cast<uint16_t*>(krow + 2 * lane) = (uint16_t)w;
        *reinterpret_cast<uint16_t*>(krow + 64 + 2 * lane) = (uint16_t)(w >> 16);
    } else {
        store_elem(a.k, krow, lane, y0);
        store_elem(a.k, krow, 32 + lane, y1);
    }
}

// Each warp loads its next token's chunks, index entry and RoPE inputs one
// token ahead.
template <int NCH, int CK, bool KF16>
__global__ void __launch_bounds__(RR_THREADS, NCH >= 4 ? 6 : 8) rmsnorm_rope_lean_kernel(const RmsRopeArgs a) {
    constexpr int DV = 256 * NCH;
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) float rr_stage[];
    float* gs = rr_stage;                 // [DV] gamma, or gamma * r
    float* stg = rr_stage + DV;           // int8 ckv: [3][DV] scale, offset, RN(1/scale)
    const int lane = threadIdx.x & 31;
    CkvDiv dv;
    const bool fold = rr_lean_stage<NCH, CK, KF16>(a, gs, stg, dv);

    const uint32_t ntok = (uint32_t)(a.B * a.S);
    const uint32_t gwarp = (blockIdx.x * RR_THREADS + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * RR_THREADS) >> 5;
    const uint32_t rowb = (uint32_t)a.D * 2u;                     // kv row bytes
    const char* xb = reinterpret_cast<const char*>(a.kv) + 16 * lane;
    const char* zb = reinterpret_cast<const char*>(a.kv) + 2 * DV + 4 * lane;
    const uint16_t* cb = a.cos + lane;
    const uint16_t* sb = a.sin + lane;
    const uint32_t nslots = (uint32_t)a.k.rows.num_slots;

    uint4 xn[NCH];
    int64_t vn = -1;
    uint32_t zn = 0u, cn = 0u, sn = 0u;
    auto fetch = [&](uint32_t t) {
        if (t >= ntok) return;
        const char* p = xb + (uint64_t)t * rowb;
#pragma unroll
        for (int m = 0; m < NCH; ++m) xn[m] = __ldg(reinterpret_cast<const uint4*>(p + 512 * m));
        vn = a.index_i64 ? __ldg(reinterpret_cast<const long long*>(a.index) + t)
                         : (int64_t)__ldg(reinterpret_cast<const int32_t*>(a.index) + t);
        zn = __ldg(reinterpret_cast<const uint32_t*>(zb + (uint64_t)t * rowb));
        const uint16_t* cp = cb + (uint64_t)t * 64u;
        const uint16_t* sp = sb + (uint64_t)t * 64u;
        cn = (uint32_t)__ldg(cp) | ((uint32_t)__ldg(cp + 32) << 16);
        sn = (uint32_t)__ldg(sp) | ((uint32_t)__ldg(sp + 32) << 16);
    };
    fetch(gwarp);
    for (uint32_t t = gwarp; t < ntok; t += nwarps) {
        uint4 xv[NCH];
#pragma unroll
        for (int m = 0; m < NCH; ++m) xv[m] = xn[m];
        const int64_t v = vn;
        const uint32_t zr = zn, cr = cn, sr = sn;
        fetch(t + nwarps);
        if (v == -1) continue;
        if (v < 0 || v >= (int64_t)nslots) {
            if (lane == 0) raise_fault(FAULT_SLOT_RANGE);
            continue;
        }
        rr_lean_token<NCH, CK, KF16>(a, xv, zr, cr, sr, (uint32_t)v, gs, stg, dv, fold, lane);
    }
}

}  // namespace kvq
