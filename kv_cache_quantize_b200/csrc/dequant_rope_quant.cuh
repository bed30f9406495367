// dequant_rope_quant.cuh -- dequant_rope_quant_kvcache kernel
// (aclnnDequantRopeQuantKvcache 算子深度解析: 计算步骤公式 steps 1-5, 两种 KV
// Cache 更新模式, Kernel 实现要点: dequant Cast -> Mul -> Muls -> Add, RoPE with
// the sine negated first, quant Div -> Add offset -> round to int8).
//
// Two kernels: the pipelined one (aligned inputs, D a multiple of 8 up to
// 256; see its comment below) and a general one for every other shape and
// alignment the pages allow (one CTA per token, one thread per RoPE pair or
// per value).
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
    int32_t out_vec8;               // q_out, k_out, v_out are 8-byte aligned
    int32_t rows_vec4;              // k / v cache rows start on 4-byte boundaries
    int32_t Nq, Nkv, D;
    uint16_t* q_out;        // [B*S, Nq*D]
    uint16_t* k_out;        // [B*S, Nkv*D] or null
    uint16_t* v_out;
    // pipelined kernel only
    int32_t tps;            // tokens per shared-memory stage
    int32_t stages;
};

__device__ __forceinline__ float dq_bias(const DrqArgs& a, int64_t i) {
    switch (a.bias_kind) {
        case 0: return reinterpret_cast<const float*>(a.bias)[i];
        case 1: return __half2float(__ushort_as_half(reinterpret_cast<const unsigned short*>(a.bias)[i]));
        case 2: return __uint_as_float((uint32_t) reinterpret_cast<const uint16_t*>(a.bias)[i] << 16);
        default: return __int2float_rn(reinterpret_cast<const int32_t*>(a.bias)[i]);
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

// ---------------------------------------------------------------------------
// General kernel: one CTA per token (grid-stride over tokens).  Thread i
// takes RoPE pairs i, i + blockDim, ... of the q and k heads -- value j of a
// head and its half-rotation partner j + D/2 together -- then values i,
// i + blockDim, ... of the v heads.  Element loads and stores are 16-bit or
// 8-bit and coalesced across the CTA; any alignment, any even D.
// ---------------------------------------------------------------------------
constexpr int DG_THREADS = 256;

// element i of the token's x row, dequantised: ((float)x * ws) * act + bias
__device__ __forceinline__ float dg_value(const DrqArgs& a, int64_t t, int64_t i, float act) {
    if (a.x_kind == 0) {
        float v = __fmul_rn(__int2float_rn(reinterpret_cast<const int32_t*>(a.x)[t * a.H + i]), a.weight_scale[i]);
        if (a.activation_scale) v = __fmul_rn(v, act);
        if (a.bias) v = __fadd_rn(v, dq_bias(a, i));
        return v;
    }
    const uint32_t h = reinterpret_cast<const uint16_t*>(a.x)[t * a.H + i];
    return a.x_kind == 2 ? __half2float(__ushort_as_half((unsigned short)h)) : __uint_as_float(h << 16);
}

__device__ __forceinline__ float dg_half(const uint16_t* p, int64_t i, bool f16) {
    const uint32_t h = p[i];
    return f16 ? __half2float(__ushort_as_half((unsigned short)h)) : __uint_as_float(h << 16);
}

__device__ __forceinline__ uint16_t dg_round16(float v, bool f16) {
    return (uint16_t)(f16 ? to_f16_bits(v) : to_bf16_bits(v));
}

// static int8 of channel c: round half to even of o / scale + offset, saturated
__device__ __forceinline__ uint8_t dg_int8(const float* sc, const float* of, int64_t c, float o) {
    float q = __fdiv_rn(o, sc[c]);
    if (of) q = __fadd_rn(q, of[c]);
    return (uint8_t)int8_rne_sat(q);
}

__global__ void __launch_bounds__(DG_THREADS) dequant_rope_quant_general_kernel(const DrqArgs a) {
    pdl_wait();
    pdl_trigger();
    const int64_t ntok = a.B * a.S;
    const int D = a.D, h = a.D / 2;
    const int64_t C = (int64_t)a.Nkv * D;
    const bool f16 = a.cos_f16 != 0;
    for (int64_t t = blockIdx.x; t < ntok; t += gridDim.x) {
        const int64_t slot = dq_slot(a, t);
        if (slot == -2 && threadIdx.x == 0) raise_fault(FAULT_SLOT_RANGE);
        uint8_t* krow = slot >= 0 ? slot_row(a.kc, slot) : nullptr;
        uint8_t* vrow = slot >= 0 ? slot_row(a.vc, slot) : nullptr;
        const float act = (a.x_kind == 0 && a.activation_scale) ? a.activation_scale[t] : 1.0f;
        const uint16_t* cs = a.cos + t * D;
        const uint16_t* sn = a.sin + t * D;
        // q and k heads: RoPE pairs (j, j + D/2)
        const int64_t npairs = (int64_t)(a.Nq + a.Nkv) * h;
        for (int64_t p = threadIdx.x; p < npairs; p += blockDim.x) {
            const int hd = (int)(p / h), j = (int)(p - (int64_t)hd * h);
            const int64_t e0 = (int64_t)hd * D + j;
            const float u0 = dg_value(a, t, e0, act), u1 = dg_value(a, t, e0 + h, act);
            // o_j = u_j c_j - u_{j+h} s_j,  o_{j+h} = u_{j+h} c_{j+h} + u_j s_{j+h}
            const float o0 = __fadd_rn(__fmul_rn(u0, dg_half(cs, j, f16)), __fmul_rn(u1, -dg_half(sn, j, f16)));
            const float o1 = __fadd_rn(__fmul_rn(u1, dg_half(cs, j + h, f16)), __fmul_rn(u0, dg_half(sn, j + h, f16)));
            if (hd < a.Nq) {
                uint16_t* q = a.q_out + t * (int64_t)a.Nq * D + e0;
                q[0] = dg_round16(o0, f16);
                q[h] = dg_round16(o1, f16);
                continue;
            }
            const int64_t c = (int64_t)(hd - a.Nq) * D + j;
            if (a.k_out) {
                a.k_out[t * C + c] = dg_round16(o0, f16);
                a.k_out[t * C + c + h] = dg_round16(o1, f16);
            }
            if (krow) {
                krow[c] = dg_int8(a.scale_k, a.offset_k, c, o0);
                krow[c + h] = dg_int8(a.scale_k, a.offset_k, c + h, o1);
            }
        }
        // v heads: no RoPE
        for (int64_t c = threadIdx.x; c < C; c += blockDim.x) {
            const float o = dg_value(a, t, (int64_t)(a.Nq + a.Nkv) * D + c, act);
            if (a.v_out) a.v_out[t * C + c] = dg_round16(o, f16);
            if (vrow) vrow[c] = dg_int8(a.scale_v, a.offset_v, c, o);
        }
    }
}

// ---------------------------------------------------------------------------
// Pipelined kernel (16-byte aligned x, cos and sin).  CTA = DT_CONSUMERS
// consumer warps + 1 producer warp.  A stage holds TPS consecutive tokens:
// their x rows, cos rows and sin rows arrive by three bulk copies (each a
// contiguous span); the producer resolves the tokens' destination slots and
// activation scales one stage ahead and stores them next to the stage.  The
// per-channel parameters (weight scale, bias, the k / v scales and offsets)
// are staged in shared memory once per CTA as binary32.
//
// Lane layout: a head of D values is L = D/8 lanes; lane l of a head holds the
// four values [4l, 4l + 4) and their half-rotation partners [D/2 + 4l,
// D/2 + 4l + 4), so RoPE needs no shuffle, and a warp holds 32/L heads side by
// side (a PASS).  Each token of a stage has 8/TPS consumer warps, which take
// its passes round-robin (spreading the costlier k / v passes with their int8
// quantisation evenly) and widen its cos / sin once.
//
// The stage count S, TPS and (for the common head size 128) D are template
// parameters (S in 2..4, TPS in 2, 4, 8: every pair the launch rule picks for
// H <= 4096; DC = 0 reads D from the arguments): with the ring's shape and the
// lane layout known at compile time the consumers' index and address
// arithmetic folds to constants, which measured 11 % faster (61.9 -> 55.3 us
// on x int32 [16, 1024, 3072]) than the same kernel reading all three from its
// arguments.
// ---------------------------------------------------------------------------
constexpr int DT_CONSUMERS = 8;
constexpr int DT_THREADS = (DT_CONSUMERS + 1) * 32;

__host__ __device__ inline uint32_t dt_header_bytes(int stages, int tps) {
    return ((uint32_t)(16 * stages + 12 * stages * tps) + 127u) & ~127u;
}

// binary32 parameters: weight scale and bias [H] (int32 x only), then the k and
// v scales, offsets and scale reciprocals [C = Nkv * D]
__host__ __device__ inline uint32_t dt_param_bytes(int64_t H, int64_t C, bool dq) {
    return (uint32_t)(((dq ? 8 * H : 0) + 24 * C + 127) & ~127);
}

__host__ __device__ inline uint32_t dt_stage_bytes(int tps, int64_t H, int x_bytes, int D) {
    return (uint32_t)(((tps * H * x_bytes + 127) & ~127) + 2 * ((tps * D * 2 + 127) & ~127));
}

// Raw index entry of token t (page mode: its slot; contiguous mode: the start
// position of its batch).
__device__ __forceinline__ int64_t dq_index_raw(const DrqArgs& a, int64_t t) {
    return load_slot(a.indices, a.indices_i64, a.cache_mode == 1 ? t : t / a.S);
}

// Destination row of token t from its raw index entry: >= 0 a cache slot,
// -1 skip, -2 bad index (the rules of dq_slot).
__device__ __forceinline__ int64_t dq_resolve(const DrqArgs& a, int64_t t, int64_t raw) {
    if (a.cache_mode == 1) {
        if (raw != -1 && !slot_ok(raw, a.kc.num_slots)) return -2;
        return raw;
    }
    const int64_t b = t / a.S, s = t - b * a.S;
    const int64_t c1 = a.kc.block_size;
    if (raw == -1) return -1;
    if (raw < 0 || raw + s >= c1 || b * c1 >= a.kc.num_slots) return -2;
    return b * c1 + raw + s;
}

// four 16-bit floats from shared memory, widened
template <bool F16>
__device__ __forceinline__ void dt_lds4h(const uint16_t* p, float (&v)[4]) {
    const uint2 q = *reinterpret_cast<const uint2*>(p);
    v[0] = F16 ? f16_lo(q.x) : bf16_lo(q.x);
    v[1] = F16 ? f16_hi(q.x) : bf16_hi(q.x);
    v[2] = F16 ? f16_lo(q.y) : bf16_lo(q.y);
    v[3] = F16 ? f16_hi(q.y) : bf16_hi(q.y);
}

__device__ __forceinline__ void dt_lds4i(const int32_t* p, float (&v)[4]) {
    const int4 q = *reinterpret_cast<const int4*>(p);
    v[0] = __int2float_rn(q.x); v[1] = __int2float_rn(q.y);
    v[2] = __int2float_rn(q.z); v[3] = __int2float_rn(q.w);
}

__device__ __forceinline__ void dt_lds4f(const float* p, float (&v)[4]) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}

__device__ __forceinline__ uint32_t dt_int8x4(const float (&o)[4], const float* sc, const float* of, const float* rc) {
    float s[4], f[4], r[4];
    dt_lds4f(sc, s);
    dt_lds4f(of, f);
    dt_lds4f(rc, r);
    return int8x4_quant(o, s, f, r);
}

// XK: 0 int32 x (dequantised), 1 bf16 x, 2 f16 x.  F16: cos / sin and the
// 16-bit outputs are f16 (else bf16).  S stages of TPS tokens (a.stages and
// a.tps hold the same values); head size DC, or a.D when DC is 0.
template <int XK, bool F16, int S, int TPS, int DC>
__global__ void __launch_bounds__(DT_THREADS) dequant_rope_quant_tma_kernel(const DrqArgs a) {
    static_assert(S >= 2 && S <= 4 && (TPS == 2 || TPS == 4 || TPS == 8), "ring shape");
    static_assert(DC == 0 || (DC % 8 == 0 && DC <= 256), "head size");
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(128) uint8_t smem[];
    const int D = DC ? DC : a.D;
    constexpr int XB = XK == 0 ? 4 : 2;
    constexpr bool DQ = XK == 0;
    const int64_t H = a.H;
    const int C = a.Nkv * D;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + S;
    int64_t* slots = reinterpret_cast<int64_t*>(empty + S);
    float* acts = reinterpret_cast<float*>(slots + S * TPS);
    float* prm = reinterpret_cast<float*>(smem + dt_header_bytes(S, TPS));
    float* p_ws = prm;                      // [H]  (int32 x)
    float* p_bias = prm + H;                // [H]  (int32 x; -0.0, the exact additive identity, when absent)
    float* p_sk = prm + (DQ ? 2 * H : 0);   // [C]
    float* p_sv = p_sk + C;
    float* p_ok = p_sv + C;                 // [C] (0 when absent)
    float* p_ov = p_ok + C;
    float* p_rk = p_ov + C;                 // [C] RN(1/scale) where the fast quotient applies, else 0
    float* p_rv = p_rk + C;
    uint8_t* stages = smem + dt_header_bytes(S, TPS) + dt_param_bytes(H, C, DQ);
    const uint32_t x_span = (uint32_t)((TPS * H * XB + 127) & ~127);
    const uint32_t cs_span = (uint32_t)((TPS * D * 2 + 127) & ~127);
    const uint32_t stage_bytes = x_span + 2 * cs_span;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t ntok = a.B * a.S;
    const int64_t ntiles = (ntok + TPS - 1) / TPS;

    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], DT_CONSUMERS);
        }
        mbar_init_fence();
    }
    if (DQ) {
        for (int64_t i = threadIdx.x; i < H; i += blockDim.x) {
            p_ws[i] = a.weight_scale[i];
            p_bias[i] = a.bias ? dq_bias(a, i) : -0.0f;
        }
    }
    for (int i = threadIdx.x; i < C; i += blockDim.x) {
        p_sk[i] = a.scale_k[i];
        p_sv[i] = a.scale_v[i];
        p_ok[i] = a.offset_k ? a.offset_k[i] : 0.0f;
        p_ov[i] = a.offset_v ? a.offset_v[i] : 0.0f;
        p_rk[i] = int8_quant_rcp(p_sk[i], p_ok[i]);
        p_rv[i] = int8_quant_rcp(p_sv[i], p_ov[i]);
    }
    __syncthreads();

    if (warp == DT_CONSUMERS) {
        // ---------------- producer ----------------
        // lane k < TPS holds token k's raw index entry and activation scale
        // for the next tile, loaded while the current tile is being issued
        auto fetch = [&](int64_t tile, int64_t& raw, float& act) {
            const int64_t t = tile * TPS + lane;
            raw = -1;
            act = 1.0f;
            if (lane < TPS && tile < ntiles && t < ntok) {
                raw = dq_index_raw(a, t);
                if (DQ && a.activation_scale) act = a.activation_scale[t];
            }
        };
        int it = 0;
        int64_t raw_next;
        float act_next;
        fetch(blockIdx.x, raw_next, act_next);
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
            const int st = it % S;
            const uint32_t round = (uint32_t)(it / S);
            const int64_t raw = raw_next;
            const float act = act_next;
            fetch(tile + gridDim.x, raw_next, act_next);
            if (!__all_sync(FULL_MASK, mbar_wait(&empty[st], (round & 1u) ^ 1u))) break;
            const int64_t t0 = tile * TPS;
            const int toks = (int)(ntok - t0 < TPS ? ntok - t0 : TPS);
            if (lane < toks) {
                int64_t slot = dq_resolve(a, t0 + lane, raw);
                if (slot == -2) {
                    raise_fault(FAULT_SLOT_RANGE);
                    slot = -1;
                }
                slots[st * TPS + lane] = slot;
                acts[st * TPS + lane] = act;
            }
            __syncwarp();
            if (lane == 0) {
                uint8_t* base = stages + (size_t)st * stage_bytes;
                const uint32_t xbytes = (uint32_t)(toks * H * XB), cbytes = (uint32_t)(toks * D * 2);
                mbar_arrive_expect_tx(&full[st], xbytes + 2 * cbytes);
                bulk_copy_g2s(base, reinterpret_cast<const uint8_t*>(a.x) + (size_t)t0 * H * XB, xbytes, &full[st]);
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
    // warp w serves token w / WPT of each stage and takes that token's passes
    // wt, wt + WPT, ... (wt = w mod WPT): each warp stays on one token, and the
    // stride mixes the costlier k / v passes evenly over the token's warps
    const int NH = a.Nq + 2 * a.Nkv;
    const int L = D >> 3;                     // lanes per head
    const int HPW = 32 / L;                   // heads per pass
    const int hl = lane / L, l = lane - hl * L;
    const bool lane_on = hl < HPW;
    const int NP = (NH + HPW - 1) / HPW;      // passes per token
    const int j0 = 4 * l, j1 = (D >> 1) + 4 * l;
    constexpr int WPT = DT_CONSUMERS / TPS;
    const int my_tok = warp / WPT, wt = warp - my_tok * WPT;
    const bool v8 = a.out_vec8 != 0, r4 = a.rows_vec4 != 0;
    auto store4h = [&](uint16_t* p, const float (&o)[4]) {
        uint32_t w0, w1;
        if (F16) {
            asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(w0) : "f"(o[1]), "f"(o[0]));
            asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(w1) : "f"(o[3]), "f"(o[2]));
        } else {
            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w0) : "f"(o[1]), "f"(o[0]));
            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w1) : "f"(o[3]), "f"(o[2]));
        }
        if (v8) *reinterpret_cast<uint2*>(p) = make_uint2(w0, w1);
        else st_b64(reinterpret_cast<uint8_t*>(p), make_uint2(w0, w1));
    };
    int it = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
        const int st = it % S;
        const uint32_t round = (uint32_t)(it / S);
        if (!__all_sync(FULL_MASK, mbar_wait(&full[st], round & 1u))) break;
        const int64_t t0 = tile * TPS;
        const int toks = (int)(ntok - t0 < TPS ? ntok - t0 : TPS);
        const uint8_t* base = stages + (size_t)st * stage_bytes;
        if (my_tok < toks && lane_on) {
            const int64_t t = t0 + my_tok;
            const int64_t slot = slots[st * TPS + my_tok];
            const float act = acts[st * TPS + my_tok];
            uint8_t* krow = slot >= 0 ? slot_row(a.kc, slot) : nullptr;
            uint8_t* vrow = slot >= 0 ? slot_row(a.vc, slot) : nullptr;
            // cos / sin at j0 (a) and j1 (b); nsa = -sin at j0
            float ca[4], cb[4], nsa[4], sb[4];
            const uint16_t* cp = reinterpret_cast<const uint16_t*>(base + x_span) + my_tok * D;
            const uint16_t* sp = reinterpret_cast<const uint16_t*>(base + x_span + cs_span) + my_tok * D;
            dt_lds4h<F16>(cp + j0, ca);
            dt_lds4h<F16>(cp + j1, cb);
            dt_lds4h<F16>(sp + j0, nsa);
            dt_lds4h<F16>(sp + j1, sb);
#pragma unroll
            for (int k = 0; k < 4; ++k) nsa[k] = -nsa[k];
            const uint8_t* xt = base + (size_t)my_tok * H * XB;
            for (int p = wt; p < NP; p += WPT) {
                const int hd = p * HPW + hl;
                if (hd >= NH) continue;
                float ua[4], ub[4];
                const int e0 = hd * D;
                if (DQ) {
                    dt_lds4i(reinterpret_cast<const int32_t*>(xt) + e0 + j0, ua);
                    dt_lds4i(reinterpret_cast<const int32_t*>(xt) + e0 + j1, ub);
                    // dequant: ((float)x * weight_scale) * activation_scale + bias
                    float wa[4], wb[4], ba[4], bb[4];
                    dt_lds4f(p_ws + e0 + j0, wa);
                    dt_lds4f(p_ws + e0 + j1, wb);
                    dt_lds4f(p_bias + e0 + j0, ba);
                    dt_lds4f(p_bias + e0 + j1, bb);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        ua[k] = __fadd_rn(__fmul_rn(__fmul_rn(ua[k], wa[k]), act), ba[k]);
                        ub[k] = __fadd_rn(__fmul_rn(__fmul_rn(ub[k], wb[k]), act), bb[k]);
                    }
                } else {
                    dt_lds4h<XK == 2>(reinterpret_cast<const uint16_t*>(xt) + e0 + j0, ua);
                    dt_lds4h<XK == 2>(reinterpret_cast<const uint16_t*>(xt) + e0 + j1, ub);
                }
                float oa[4], ob[4];
                if (hd < a.Nq + a.Nkv) {
                    // RoPE, half rotation: o_j = u_j c_j - u_{j+D/2} s_j, o_{j+D/2} = u_{j+D/2} c_{j+D/2} + u_j s_{j+D/2}
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        oa[k] = __fadd_rn(__fmul_rn(ua[k], ca[k]), __fmul_rn(ub[k], nsa[k]));
                        ob[k] = __fadd_rn(__fmul_rn(ub[k], cb[k]), __fmul_rn(ua[k], sb[k]));
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        oa[k] = ua[k];
                        ob[k] = ub[k];
                    }
                }
                if (hd < a.Nq) {
                    uint16_t* q = a.q_out + t * (int64_t)(a.Nq * D) + e0;
                    store4h(q + j0, oa);
                    store4h(q + j1, ob);
                    continue;
                }
                const bool is_k = hd < a.Nq + a.Nkv;
                const int c0 = (is_k ? hd - a.Nq : hd - a.Nq - a.Nkv) * D;   // channel base in [0, Nkv*D)
                if (a.k_out) {
                    uint16_t* kv = (is_k ? a.k_out : a.v_out) + t * (int64_t)C + c0;
                    store4h(kv + j0, oa);
                    store4h(kv + j1, ob);
                }
                uint8_t* row = is_k ? krow : vrow;
                if (row == nullptr) continue;
                const float* sc = (is_k ? p_sk : p_sv) + c0;
                const float* of = (is_k ? p_ok : p_ov) + c0;
                const float* rc = (is_k ? p_rk : p_rv) + c0;
                const uint32_t q0 = dt_int8x4(oa, sc + j0, of + j0, rc + j0);
                const uint32_t q1 = dt_int8x4(ob, sc + j1, of + j1, rc + j1);
                if (r4) {
                    *reinterpret_cast<uint32_t*>(row + c0 + j0) = q0;
                    *reinterpret_cast<uint32_t*>(row + c0 + j1) = q1;
                } else {
                    st_b32(row + c0 + j0, q0);
                    st_b32(row + c0 + j1, q1);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }
}

}  // namespace kvq
