// dequant_rope_quant.cuh -- dequant_rope_quant_kvcache kernel
// (aclnnDequantRopeQuantKvcache 算子深度解析: 计算步骤公式 steps 1-5, 两种 KV
// Cache 更新模式, Kernel 实现要点: dequant Cast -> Mul -> Muls -> Add, RoPE with
// the sine negated first, quant Div -> Add offset -> round to int8).
//
// A CTA walks tokens (grid-stride); its DQ_WARPS warps split the token's
// Nq + 2*Nkv heads (warp w takes heads w, w + DQ_WARPS, ...).  Within a head of
// D values each lane holds E = D/32 consecutive values, so the first half of
// the head sits in lanes 0-15 and the second half in lanes 16-31 at the same
// register positions: the half-rotation partner of every value is one
// __shfl_xor(16) away.  Up to DQ_PASS of a warp's heads are loaded before
// any of them is processed.
#pragma once

#include "kvq_device.cuh"
#include "tma_pipe.cuh"

namespace kvq {

struct DrqArgs {
    const void* x;          // [B*S, H]
    int32_t x_kind;         // 0 int32, 1 bf16, 2 f16
    int32_t x_vec;          // x is 16-byte aligned (vector loads of int32 values)
    int64_t B, S, H;
    const uint16_t* cos;    // [B*S, D]
    const uint16_t* sin;
    int32_t cos_f16;        // cos/sin and the 16-bit outputs are f16 (else bf16)
    PagedRows kc, vc;       // rows of Nkv*D int8
    const void* indices;
    int32_t indices_i64;
    int32_t cache_mode;     // 0 contiguous, 1 page
    const float* scale_k;
    const float* scale_v;
    const float* offset_k;  // nullable
    const float* offset_v;
    const float* weight_scale;      // [H], int32 x only
    const float* activation_scale;  // [B*S] nullable
    const void* bias;               // [H] nullable
    int32_t bias_kind;              // 0 f32, 1 f16, 2 bf16, 3 int32
    int32_t params_vec;             // all f32 parameter tensors are 16-byte aligned
    int32_t Nq, Nkv, D;
    uint16_t* q_out;        // [B*S, Nq*D]
    uint16_t* k_out;        // [B*S, Nkv*D] or null
    uint16_t* v_out;
    // pipelined kernel only
    int32_t tps;            // tokens per shared-memory stage
    int32_t stages;
};

constexpr int DQ_WARPS = 8;
constexpr int DQ_MAX_HEADS_PER_WARP = 8;
constexpr int DQ_PASS = 4;

template <int E>
__device__ __forceinline__ void dq_load(const DrqArgs& a, int64_t e0, float (&u)[E], const int32_t* xi) {
    if (a.x_kind == 0) {
        int32_t v[E];
        if (E % 4 == 0 && a.x_vec) {
#pragma unroll
            for (int k = 0; k < E; k += 4) {
                const int4 w = __ldcs(reinterpret_cast<const int4*>(xi + e0 + k));
                v[k] = w.x; v[k + 1] = w.y; v[k + 2] = w.z; v[k + 3] = w.w;
            }
        } else if (E % 2 == 0 && a.x_vec) {
#pragma unroll
            for (int k = 0; k < E; k += 2) {
                const int2 w = __ldcs(reinterpret_cast<const int2*>(xi + e0 + k));
                v[k] = w.x; v[k + 1] = w.y;
            }
        } else {
#pragma unroll
            for (int k = 0; k < E; ++k) v[k] = __ldcs(xi + e0 + k);
        }
#pragma unroll
        for (int k = 0; k < E; ++k) u[k] = __int2float_rn(v[k]);
    } else {
        const uint16_t* xh = reinterpret_cast<const uint16_t*>(a.x);
#pragma unroll
        for (int k = 0; k < E; ++k) {
            const uint32_t hb = __ldcs(xh + e0 + k);
            u[k] = a.x_kind == 2 ? __half2float(__ushort_as_half((unsigned short)hb)) : __uint_as_float(hb << 16);
        }
    }
}

__device__ __forceinline__ float dq_bias(const DrqArgs& a, int64_t i) {
    switch (a.bias_kind) {
        case 0: return reinterpret_cast<const float*>(a.bias)[i];
        case 1: return __half2float(__ushort_as_half(reinterpret_cast<const unsigned short*>(a.bias)[i]));
        case 2: return __uint_as_float((uint32_t) reinterpret_cast<const uint16_t*>(a.bias)[i] << 16);
        default: return __int2float_rn(reinterpret_cast<const int32_t*>(a.bias)[i]);
    }
}

// E consecutive binary32 parameters starting at p (16-byte vectors when E % 4 == 0
// and p is 16-byte aligned, which holds for the kernels' channel offsets when the
// parameter tensors are 16-byte aligned: params_vec).
template <int E>
__device__ __forceinline__ void dq_param(const float* p, bool vec, float (&v)[E]) {
    if (E % 4 == 0 && vec) {
#pragma unroll
        for (int k = 0; k < E; k += 4) {
            const float4 w = __ldg(reinterpret_cast<const float4*>(p + k));
            v[k] = w.x; v[k + 1] = w.y; v[k + 2] = w.z; v[k + 3] = w.w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < E; ++k) v[k] = __ldg(p + k);
    }
}

__device__ __forceinline__ uint32_t dq_round16(const DrqArgs& a, float v) {
    return a.cos_f16 ? to_f16_bits(v) : to_bf16_bits(v);
}

// E 16-bit outputs, packed into 4- or 8-byte stores
template <int E>
__device__ __forceinline__ void dq_store16(uint16_t* p, const DrqArgs& a, const float (&o)[E]) {
    if (E % 4 == 0) {
#pragma unroll
        for (int k = 0; k < E; k += 4) {
            const uint2 w = make_uint2(dq_round16(a, o[k]) | (dq_round16(a, o[k + 1]) << 16),
                                       dq_round16(a, o[k + 2]) | (dq_round16(a, o[k + 3]) << 16));
            st_b64(reinterpret_cast<uint8_t*>(p + k), w);
        }
    } else if (E % 2 == 0) {
#pragma unroll
        for (int k = 0; k < E; k += 2)
            st_b32(reinterpret_cast<uint8_t*>(p + k), dq_round16(a, o[k]) | (dq_round16(a, o[k + 1]) << 16));
    } else {
#pragma unroll
        for (int k = 0; k < E; ++k) p[k] = (uint16_t)dq_round16(a, o[k]);
    }
}

// One head of one token: dequant, RoPE (q and k heads), outputs, int8 quant
// and the cache write.  Called with the whole warp (the RoPE shuffle).
template <int E>
__device__ __forceinline__ void dq_head(const DrqArgs& a, int64_t t, int hd, float (&u)[E], const float (&cs)[E],
                                        const float (&sn)[E], float act, int64_t slot, int pos, bool second_half) {
    const int D = a.D;
    const int ch0 = hd * D + pos;    // channel index within H
    const bool pv = a.params_vec != 0;
    // 1 dequant: ((float)x * weight_scale) * activation_scale + bias
    if (a.x_kind == 0) {
        float ws[E];
        dq_param<E>(a.weight_scale + ch0, pv, ws);
        float bs[E];
        if (a.bias && a.bias_kind == 0) {
            dq_param<E>(reinterpret_cast<const float*>(a.bias) + ch0, pv, bs);
        } else if (a.bias) {
#pragma unroll
            for (int k = 0; k < E; ++k) bs[k] = dq_bias(a, ch0 + k);
        }
#pragma unroll
        for (int k = 0; k < E; ++k) {
            float v = __fmul_rn(u[k], ws[k]);
            if (a.activation_scale) v = __fmul_rn(v, act);
            if (a.bias) v = __fadd_rn(v, bs[k]);
            u[k] = v;
        }
    }
    float o[E];
    if (hd < a.Nq + a.Nkv) {
        // 3 RoPE, half rotation: the partner value is 16 lanes away
#pragma unroll
        for (int k = 0; k < E; ++k) {
            const float p = __shfl_xor_sync(FULL_MASK, u[k], 16);
            const float sgn_s = second_half ? sn[k] : -sn[k];
            o[k] = __fadd_rn(__fmul_rn(u[k], cs[k]), __fmul_rn(p, sgn_s));
        }
    } else {
#pragma unroll
        for (int k = 0; k < E; ++k) o[k] = u[k];
    }
    if (hd < a.Nq) {
        dq_store16<E>(a.q_out + t * (int64_t)(a.Nq * D) + ch0, a, o);
        return;
    }
    const bool is_k = hd < a.Nq + a.Nkv;
    const int c0 = (is_k ? hd - a.Nq : hd - a.Nq - a.Nkv) * D + pos;   // channel in [0, Nkv*D)
    if (a.k_out) dq_store16<E>((is_k ? a.k_out : a.v_out) + t * (int64_t)(a.Nkv * D) + c0, a, o);
    if (slot < 0) return;
    // 4 quant: int8(rint(w / scale + offset)), saturating
    float sc[E], of[E];
    dq_param<E>((is_k ? a.scale_k : a.scale_v) + c0, pv, sc);
    const float* ofp = is_k ? a.offset_k : a.offset_v;
    if (ofp) dq_param<E>(ofp + c0, pv, of);
    uint32_t packed[(E + 3) / 4];
#pragma unroll
    for (int k = 0; k < (E + 3) / 4; ++k) packed[k] = 0u;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        float q = __fdiv_rn(o[k], sc[k]);
        if (ofp) q = __fadd_rn(q, of[k]);
        packed[k / 4] |= ((uint32_t)int8_rne_sat(q) & 0xffu) << (8 * (k % 4));
    }
    // 5 cache write
    uint8_t* row = slot_row(is_k ? a.kc : a.vc, slot) + c0;
    if (E % 4 == 0) {
#pragma unroll
        for (int k = 0; k < E / 4; ++k) st_b32(row + 4 * k, packed[k]);
    } else {
#pragma unroll
        for (int k = 0; k < E; ++k) row[k] = (uint8_t)(packed[k / 4] >> (8 * (k % 4)));
    }
}

// Destination row of token t: >= 0 a cache slot, -1 skip, -2 bad index.
__device__ __forceinline__ int64_t dq_slot(const DrqArgs& a, int64_t t) {
    if (a.cache_mode == 1) {
        const int64_t slot = load_slot(a.indices, a.indices_i64, t);
        if (slot != -1 && !slot_ok(slot, a.kc.num_slots)) return -2;
        return slot;
    }
    const int64_t b = t / a.S, s = t - b * a.S;
    const int64_t start = load_slot(a.indices, a.indices_i64, b);
    const int64_t c1 = a.kc.block_size;
    if (start == -1) return -1;
    if (start < 0 || start + s >= c1 || b * c1 >= a.kc.num_slots) return -2;
    return b * c1 + start + s;
}

__device__ __forceinline__ float half_bits_to_f32(uint32_t h, bool f16) {
    return f16 ? __half2float(__ushort_as_half((unsigned short)h)) : __uint_as_float(h << 16);
}

template <int E>
__global__ void __launch_bounds__(DQ_WARPS * 32) dequant_rope_quant_kernel(const DrqArgs a) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int NH = a.Nq + 2 * a.Nkv;
    const int64_t ntok = a.B * a.S;
    const int D = a.D;
    const int pos = lane * E;                // first position of this lane inside a head
    const bool second_half = lane >= 16;
    const int32_t* xi = reinterpret_cast<const int32_t*>(a.x);

    for (int64_t t = blockIdx.x; t < ntok; t += gridDim.x) {
        // destination row of this token (or -1 skip / -2 fault)
        const int64_t slot = dq_slot(a, t);
        if (slot == -2 && threadIdx.x == 0) raise_fault(FAULT_SLOT_RANGE);

        float cs[E], sn[E];
#pragma unroll
        for (int k = 0; k < E; ++k) {
            const uint32_t cb = a.cos[t * D + pos + k], sb = a.sin[t * D + pos + k];
            cs[k] = a.cos_f16 ? __half2float(__ushort_as_half((unsigned short)cb)) : __uint_as_float(cb << 16);
            sn[k] = a.cos_f16 ? __half2float(__ushort_as_half((unsigned short)sb)) : __uint_as_float(sb << 16);
        }
        const float act = (a.x_kind == 0 && a.activation_scale) ? a.activation_scale[t] : 1.0f;

        // the warp's heads are hd = warp + i * DQ_WARPS; DQ_PASS of them are
        // loaded before any is processed
        const int nh = (NH - warp + DQ_WARPS - 1) / DQ_WARPS;
        for (int i0 = 0; i0 < nh; i0 += DQ_PASS) {
            float u[DQ_PASS][E];
#pragma unroll
            for (int i = 0; i < DQ_PASS; ++i) {
                const int hd = warp + (i0 + i) * DQ_WARPS;
                if (i0 + i < nh) dq_load<E>(a, t * a.H + (int64_t)hd * D + pos, u[i], xi);
            }
#pragma unroll
            for (int i = 0; i < DQ_PASS; ++i) {
                if (i0 + i >= nh) break;
                const int hd = warp + (i0 + i) * DQ_WARPS;
                dq_head<E>(a, t, hd, u[i], cs, sn, act, slot, pos, second_half);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Pipelined kernel (16-byte aligned x, cos and sin).  CTA = DQ_WARPS consumer
// warps + 1 producer warp.  A stage holds TPS consecutive tokens: their x rows,
// cos rows and sin rows arrive by three bulk copies (each a contiguous span),
// and the producer stores their destination slots next to them.  Consumers
// keep the head mapping of the direct kernel and read x, cos and sin from
// shared memory.
// ---------------------------------------------------------------------------
constexpr int DT_THREADS = (DQ_WARPS + 1) * 32;

__host__ __device__ inline uint32_t dt_header_bytes(int stages, int tps) {
    return ((uint32_t)(16 * stages + 8 * stages * tps) + 127u) & ~127u;
}

__host__ __device__ inline uint32_t dt_stage_bytes(int tps, int64_t H, int x_bytes, int D) {
    return (uint32_t)(((tps * H * x_bytes + 127) & ~127) + 2 * ((tps * D * 2 + 127) & ~127));
}

template <int E>
__global__ void __launch_bounds__(DT_THREADS) dequant_rope_quant_tma_kernel(const DrqArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int S = a.stages, TPS = a.tps, D = a.D;
    const int xb = a.x_kind == 0 ? 4 : 2;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + S;
    int64_t* slots = reinterpret_cast<int64_t*>(empty + S);
    uint8_t* stages = smem + dt_header_bytes(S, TPS);
    const uint32_t x_span = (uint32_t)((TPS * a.H * xb + 127) & ~127);
    const uint32_t cs_span = (uint32_t)((TPS * D * 2 + 127) & ~127);
    const uint32_t stage_bytes = x_span + 2 * cs_span;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t ntok = a.B * a.S;
    const int64_t ntiles = (ntok + TPS - 1) / TPS;

    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], DQ_WARPS);
        }
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == DQ_WARPS) {
        // ---------------- producer ----------------
        int it = 0;
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
            const int st = it % S;
            const uint32_t round = (uint32_t)(it / S);
            if (!__all_sync(FULL_MASK, mbar_wait(&empty[st], (round & 1u) ^ 1u))) break;
            const int64_t t0 = tile * TPS;
            const int toks = (int)(ntok - t0 < TPS ? ntok - t0 : TPS);
            for (int k = lane; k < toks; k += 32) {
                int64_t slot = dq_slot(a, t0 + k);
                if (slot == -2) {
                    raise_fault(FAULT_SLOT_RANGE);
                    slot = -1;
                }
                slots[st * TPS + k] = slot;
            }
            __syncwarp();
            if (lane == 0) {
                uint8_t* base = stages + (size_t)st * stage_bytes;
                const uint32_t xbytes = (uint32_t)(toks * a.H * xb), cbytes = (uint32_t)(toks * D * 2);
                mbar_arrive_expect_tx(&full[st], xbytes + 2 * cbytes);
                bulk_copy_g2s(base, reinterpret_cast<const uint8_t*>(a.x) + (size_t)t0 * a.H * xb, xbytes, &full[st]);
                bulk_copy_g2s(base + x_span, a.cos + (size_t)t0 * D, cbytes, &full[st]);
                bulk_copy_g2s(base + x_span + cs_span, a.sin + (size_t)t0 * D, cbytes, &full[st]);
            }
            __syncwarp();
        }
        if (lane == 0)
            for (int k = it > S ? it - S : 0; k < it; ++k) mbar_wait(&full[k % S], (uint32_t)(k / S) & 1u);
        return;
    }

    // ---------------- consumers ----------------
    const int NH = a.Nq + 2 * a.Nkv;
    const int pos = lane * E;
    const bool second_half = lane >= 16;
    const bool f16 = a.cos_f16 != 0;
    const int nh = (NH - warp + DQ_WARPS - 1) / DQ_WARPS;
    int it = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
        const int st = it % S;
        const uint32_t round = (uint32_t)(it / S);
        if (!__all_sync(FULL_MASK, mbar_wait(&full[st], round & 1u))) break;
        const int64_t t0 = tile * TPS;
        const int toks = (int)(ntok - t0 < TPS ? ntok - t0 : TPS);
        const uint8_t* base = stages + (size_t)st * stage_bytes;
        for (int k = 0; k < toks; ++k) {
            const int64_t t = t0 + k;
            const int64_t slot = slots[st * TPS + k];
            const uint16_t* cw = reinterpret_cast<const uint16_t*>(base + x_span) + k * D + pos;
            const uint16_t* sw = reinterpret_cast<const uint16_t*>(base + x_span + cs_span) + k * D + pos;
            float cs[E], sn[E];
            if (E % 4 == 0) {
#pragma unroll
                for (int e = 0; e < E; e += 4) {
                    const uint2 c2 = *reinterpret_cast<const uint2*>(cw + e);
                    const uint2 s2 = *reinterpret_cast<const uint2*>(sw + e);
                    cs[e] = half_bits_to_f32(c2.x & 0xffffu, f16); cs[e + 1] = half_bits_to_f32(c2.x >> 16, f16);
                    cs[e + 2] = half_bits_to_f32(c2.y & 0xffffu, f16); cs[e + 3] = half_bits_to_f32(c2.y >> 16, f16);
                    sn[e] = half_bits_to_f32(s2.x & 0xffffu, f16); sn[e + 1] = half_bits_to_f32(s2.x >> 16, f16);
                    sn[e + 2] = half_bits_to_f32(s2.y & 0xffffu, f16); sn[e + 3] = half_bits_to_f32(s2.y >> 16, f16);
                }
            } else {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    cs[e] = half_bits_to_f32(cw[e], f16);
                    sn[e] = half_bits_to_f32(sw[e], f16);
                }
            }
            const float act = (a.x_kind == 0 && a.activation_scale) ? a.activation_scale[t] : 1.0f;
            for (int i = 0; i < nh; ++i) {
                const int hd = warp + i * DQ_WARPS;
                float u[E];
                const int64_t e0 = (int64_t)k * a.H + (int64_t)hd * D + pos;
                if (a.x_kind == 0) {
                    const int32_t* xi = reinterpret_cast<const int32_t*>(base) + e0;
                    if (E % 4 == 0) {
#pragma unroll
                        for (int e = 0; e < E; e += 4) {
                            const int4 w = *reinterpret_cast<const int4*>(xi + e);
                            u[e] = __int2float_rn(w.x); u[e + 1] = __int2float_rn(w.y);
                            u[e + 2] = __int2float_rn(w.z); u[e + 3] = __int2float_rn(w.w);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < E; ++e) u[e] = __int2float_rn(xi[e]);
                    }
                } else {
                    const uint16_t* xh = reinterpret_cast<const uint16_t*>(base) + e0;
#pragma unroll
                    for (int e = 0; e < E; ++e) u[e] = half_bits_to_f32(xh[e], a.x_kind == 2);
                }
                dq_head<E>(a, t, hd, u, cs, sn, act, slot, pos, second_half);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }
}

}  // namespace kvq
