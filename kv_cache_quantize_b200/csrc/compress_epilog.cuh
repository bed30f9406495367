// compress_epilog.cuh -- kv_compress_epilog kernel (aclnnKvCompressEpilog,
// 计算公式 scenarios 1-3 and 约束说明 for the packed-row size).
//
// Work decomposition.  A row of d 16-bit values (bf16; f16 is accepted in
// modes 0/1, whose rope is copied as it is) is d/64 SEGMENTS of 64 values:
// the (d-64)/64 nope segments and the rope segment last.  A segment is handled
// by a TEAM of 8 lanes, each lane one 16-byte chunk of 8 values, so a warp
// works on 4 segments at a time and a 64-value quantisation group is one team
// (FP4 groups of 32 / 16 are 4 / 2 lanes of it).  A warp owns a tile of up to
// 8 consecutive rows (ce_rows, picked by the host): its first lanes load the
// tile's slots once (coalesced), the teams walk the tile's segments, and
// CE_UNROLL segments per team are loaded before any is processed so each lane
// keeps several 16-byte loads in flight.
// Group maxima are butterfly shuffles inside the team.  Every output byte of a
// row has exactly one writer: codes by their chunk's lane, a group's scale by
// the group's first lane, the rope and the zero padding by the rope team.
#pragma once

#include "kvq_device.cuh"
#include "tma_pipe.cuh"

namespace kvq {

struct CompressArgs {
    const uint16_t* x;      // bf16 bit patterns (f16 in modes 0/1 when the kernel's F16 is set)
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
    // direct kernel only
    int32_t ce_rows;        // rows per warp tile, 1 .. CE_TILE
    // pipelined kernel only
    int32_t stages;         // ring depth
    int32_t ncw;            // consumer warps
    int32_t rows_aligned;   // every cache row starts on a 16-byte boundary
    int32_t bulk_out;       // packed rows leave by bulk copy (aligned rows, kvCacheCol % 16 == 0, one segment
                            // per warp, and in modes 0/1 kvCacheCol <= 2(d-64) so the input rope lies past
                            // the packed row in shared memory)
};

// Division of a code's numerator by the group scale: the one-step Markstein
// form on pairs (div_scale8 / div_scale1_x2 in kvq_device.cuh), whose E4M3 /
// E2M1 codes kvq_selftest shows equal to those of IEEE division on its whole
// domain.

// Direct kernel: a warp takes tiles of ce_rows rows (at most CE_TILE), loading
// CE_UNROLL 16-byte chunks per lane per round; the host picks the smallest
// tile whose segments still fill one round, so that a decode-sized batch is
// spread over as many warps as it has rows and each warp makes one
// load-compute-store round trip.
constexpr int CE_TILE = 8;
constexpr int CE_UNROLL = 3;
constexpr int CE_THREADS = 256;

__device__ __forceinline__ uint4 ld_scalar8(const uint16_t* p) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = (uint32_t)__ldcs(p + 2 * i) | ((uint32_t)__ldcs(p + 2 * i + 1) << 16);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// One segment.  All lanes call this (the shuffles need the whole warp); lanes
// whose segment is inactive or skipped carry live == false.
// x_i / sf for the eight values of a lane: Markstein-corrected multiply by the
// reciprocal when the scale is in the self-tested range, IEEE division else.
__device__ __forceinline__ void div_by_scale8(const float (&f)[8], float sf, float (&q)[8]) {
    if (scale_in_fast_range(sf)) {
        const float r = __frcp_rn(sf);
        div_scale8(f, sf, r, q);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(f[i], sf);
    }
}

// One segment of 64 values, one 16-byte chunk per lane of an 8-lane team.
// All lanes call this (the shuffles need the whole warp); row == nullptr for
// lanes whose segment is inactive or whose token is skipped.
template <int MODE, int G, bool F16>
__device__ __forceinline__ void ce_segment(const CompressArgs& a, const uint4& v, uint8_t* row, int j, int sub) {
    constexpr int GL = (MODE == 2 ? G : 64) / 8;   // lanes per quantisation group
    uint32_t m = absmax_bits8(v);
    if (GL >= 2) m = max(m, __shfl_xor_sync(FULL_MASK, m, 1));
    if (GL >= 4) m = max(m, __shfl_xor_sync(FULL_MASK, m, 2));
    if (GL >= 8) m = max(m, __shfl_xor_sync(FULL_MASK, m, 4));
    if (row == nullptr) return;

    const bool rope = (j == a.nseg - 1);
    float f[8];
    widen8<F16>(v, f);
    const float amax = half_value<F16>(m);

    if (MODE == 0) {
        if (!rope) {
            // scale_g = amax / FP8_MAX, stored as bf16; codes use the stored scale
            const uint32_t sb = to_bf16_bits(div_by_fmax(amax, 448.0f));
            const float sf = __uint_as_float(sb << 16);
            uint2 codes = make_uint2(0u, 0u);
            if (sf != 0.0f) {
                float q[8];
                div_by_scale8(f, sf, q);
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
            const uint32_t b = e8m0_ceil(div_by_fmax(amax, 448.0f));
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
            const uint32_t sb = to_bf16_bits(div_by_fmax(amax, 6.0f));
            const float sf = __uint_as_float(sb << 16);
            uint32_t codes = 0u;
            if (sf != 0.0f) {
                float q[8];
                div_by_scale8(f, sf, q);
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

template <int MODE, int G, bool F16>
__global__ void __launch_bounds__(CE_THREADS) compress_epilog_kernel(const CompressArgs a) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int team = lane >> 3;
    const int sub = lane & 7;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int tr = a.ce_rows;
    const int64_t ntiles = (a.T + tr - 1) / tr;

    for (int64_t tile = gwarp; tile < ntiles; tile += nwarps) {
        const int64_t row0 = tile * tr;
        const int rows = (int)(a.T - row0 < tr ? a.T - row0 : tr);
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
            for (int u = 0; u < CE_UNROLL; ++u)
                ce_segment<MODE, G, F16>(a, v[u], live[u] ? slot_row(a.cache, sl[u]) : nullptr, jj[u], sub);
        }
    }
}

// ---------------------------------------------------------------------------
// Pipelined kernel (16-byte aligned rows).  A stage holds a tile of 32 rows,
// brought into shared memory by the producer warp with one bulk copy per
// valid row (skipped rows are never read); their destination row pointers sit
// next to the stage.  Consumer warp w owns the 64-value segment columns
// j = w, w + NCW, ... of the tile and lane r owns row r, so every lane
// quantises whole 64-value groups on its own (no shuffles) and the nope /
// rope branch is uniform across a warp.  Shared-memory rows are padded by 16
// bytes, which spreads the 32 lanes' 16-byte reads over all banks.
// ---------------------------------------------------------------------------
constexpr int CT_ROWS = 32;
constexpr int CT_MAX_CONSUMER_WARPS = 16;
constexpr int CT_MAX_THREADS = (CT_MAX_CONSUMER_WARPS + 1) * 32;

__host__ __device__ inline uint32_t ct_header_bytes(int stages) {
    return ((uint32_t)(16 * stages + 8 + 8 * stages * CT_ROWS) + 127u) & ~127u;
}

__host__ __device__ inline uint32_t ct_pitch(int nseg) { return (uint32_t)nseg * 128u + 16u; }

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

// |x| maximum of the bf16 (or f16) values of nchunks 16-byte chunks (as bits)
template <bool F16>
__device__ __forceinline__ uint32_t seg_absmax_bits(const uint8_t* seg, int nchunks) {
    uint32_t m2 = 0u;
    for (int k = 0; k < nchunks; ++k) {
        const uint4 v = lds128(seg + 16 * k);
        if (F16) m2 = absmax_f16x2(m2, absmax_f16x2(absmax_f16x2(v.x, v.y), absmax_f16x2(v.z, v.w)));
        else m2 = absmax_bf16x2(m2, absmax_bf16x2(absmax_bf16x2(v.x, v.y), absmax_bf16x2(v.z, v.w)));
    }
    m2 &= 0x7fff7fffu;
    return max(m2 & 0xffffu, m2 >> 16);
}

// Codes of eight values divided by the scale sf through the negated one-step
// quotient (div_scale1_neg_x2): FP8 E4M3 as two words, or FP4 E2M1 as one.
__device__ __forceinline__ uint2 e4m3x8_div(const float (&f)[8], float sf, float r) {
    float t[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) div_scale1_neg_x2(f[i], f[i + 1], sf, r, t[i], t[i + 1]);
    const uint2 c = fp8x8<false>(t);
    return make_uint2(c.x ^ 0x80808080u, c.y ^ 0x80808080u);
}

__device__ __forceinline__ uint32_t e2m1x8_div(const float (&f)[8], float sf, float r) {
    float t[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) div_scale1_neg_x2(f[i], f[i + 1], sf, r, t[i], t[i + 1]);
    return e2m1x8(t) ^ 0x88888888u;
}

// Outputs of one 64-value segment held in registers: the code bytes packed
// little-endian in 32-bit words, and the segment's scale bits (mode 0: one
// bf16, mode 1: one E8M0 byte, mode 2: 64/G bf16 packed).  The bf16 rope of
// modes 0/1 is copied, not computed, and never lands here.
struct SegOut {
    uint32_t w[16];
    uint32_t sc[2];
};

// Number of output words of a computed segment.
template <int MODE, int G>
__device__ __forceinline__ int seg_words(bool rope) {
    if (rope) return 16;
    return MODE == 2 ? 8 : 16;
}

template <int MODE, int G, bool F16>
__device__ __forceinline__ void ct_compute_nope(const uint8_t* seg, SegOut& o) {
    if (MODE == 0 || MODE == 1) {
        const float amax = half_value<F16>(seg_absmax_bits<F16>(seg, 8));
        float sf, r = 0.0f;
        bool fast = true;
        if (MODE == 0) {
            o.sc[0] = to_bf16_bits(div_by_fmax(amax, 448.0f));
            sf = __uint_as_float(o.sc[0] << 16);
            fast = scale_in_fast_range(sf);
            if (fast) r = __frcp_rn(sf);
        } else {
            o.sc[0] = e8m0_ceil(div_by_fmax(amax, 448.0f));
            sf = e8m0_reciprocal(o.sc[0]);      // multiplier 2^(127-b)
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            float f[8], q[8];
            widen8<F16>(lds128(seg + 16 * k), f);
            if (MODE == 1) {
#pragma unroll
                for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(f[i], sf);
            } else if (sf == 0.0f) {
#pragma unroll
                for (int i = 0; i < 8; ++i) q[i] = 0.0f;
            } else if (fast) {
                const uint2 c = e4m3x8_div(f, sf, r);
                o.w[2 * k] = c.x;
                o.w[2 * k + 1] = c.y;
                continue;
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(f[i], sf);
            }
            const uint2 c = fp8x8<false>(q);
            o.w[2 * k] = c.x;
            o.w[2 * k + 1] = c.y;
        }
    } else {
        constexpr int GC = G / 8;                   // chunks per group
        constexpr int NG = 64 / G;                  // groups per segment
        uint32_t sb[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const uint8_t* gseg = seg + g * G * 2;
            const float amax = __uint_as_float(seg_absmax_bits<false>(gseg, GC) << 16);
            sb[g] = to_bf16_bits(div_by_fmax(amax, 6.0f));
            const float sf = __uint_as_float(sb[g] << 16);
            const bool fast = scale_in_fast_range(sf);
            const float r = fast ? __frcp_rn(sf) : 0.0f;
#pragma unroll
            for (int k = 0; k < GC; ++k) {
                float f[8], q[8];
                widen8<false>(lds128(gseg + 16 * k), f);
                if (sf == 0.0f) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) q[i] = 0.0f;
                } else if (fast) {
                    o.w[g * GC + k] = e2m1x8_div(f, sf, r);
                    continue;
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(f[i], sf);
                }
                o.w[g * GC + k] = e2m1x8(q);
            }
        }
        o.sc[0] = sb[0] | (sb[1] << 16);
        o.sc[1] = sb[2] | (sb[3] << 16);
    }
}

// Mode 2 rope: static FP8 E4M3 of x * xScale, 64 bytes.
__device__ __forceinline__ void ct_compute_rope2(const CompressArgs& a, const uint8_t* seg, SegOut& o) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        float f[8], q[8];
        widen8<false>(lds128(seg + 16 * k), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(f[i], a.x_scale);
        const uint2 c = fp8x8<false>(q);
        o.w[2 * k] = c.x;
        o.w[2 * k + 1] = c.y;
    }
}

// Modes 0/1: the rope segment is kept as bf16 -- copy its 128 bytes.
template <bool SMEM>
__device__ __forceinline__ void ct_copy_rope(const uint8_t* src, uint8_t* dst, bool aligned) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (SMEM || aligned) *reinterpret_cast<uint4*>(dst + 16 * k) = lds128(src + 16 * k);
        else st_b128(dst + 16 * k, lds128(src + 16 * k));
    }
}

// Byte offsets inside the packed row.
template <int MODE, int G>
__device__ __forceinline__ int seg_code_offset(const CompressArgs& a, int j, bool rope) {
    if (rope) return MODE == 2 ? a.n / 2 : a.n;
    return MODE == 2 ? j * 32 : j * 64;
}

template <int MODE, int G>
__device__ __forceinline__ int seg_scale_offset(const CompressArgs& a, int j) {
    return MODE == 0 ? a.n + 128 + 2 * j : (MODE == 1 ? a.n + 128 + j : a.n / 2 + 64 + 2 * j * (64 / G));
}

// Write a segment's outputs to a packed row; SMEM: the row is this CTA's
// shared memory (16-byte aligned), else global memory (aligned: the row
// starts on a 16-byte boundary).
// rope_src: the input rope segment (modes 0/1 copy it to the row).
template <int MODE, int G, bool SMEM>
__device__ __forceinline__ void ct_write(const CompressArgs& a, uint8_t* row, int j, bool rope, const SegOut& o,
                                         const uint8_t* rope_src, bool aligned) {
    uint8_t* dst = row + seg_code_offset<MODE, G>(a, j, rope);
    if (rope && MODE != 2) {
        ct_copy_rope<SMEM>(rope_src, dst, aligned);
    } else {
        const int nw = seg_words<MODE, G>(rope);
#pragma unroll
        for (int k = 0; k < 16; k += 4) {
            if (k >= nw) break;
            const uint4 v = make_uint4(o.w[k], o.w[k + 1], o.w[k + 2], o.w[k + 3]);
            if (SMEM || aligned) *reinterpret_cast<uint4*>(dst + 4 * k) = v;
            else st_b128(dst + 4 * k, v);
        }
    }
    if (!rope) {
        uint8_t* sdst = row + seg_scale_offset<MODE, G>(a, j);
        if (MODE == 0 || (MODE == 2 && G == 64)) {
            if (SMEM) *reinterpret_cast<uint16_t*>(sdst) = (uint16_t)o.sc[0];
            else st_b16(sdst, o.sc[0]);
        } else if (MODE == 1) {
            *sdst = (uint8_t)o.sc[0];
        } else if (G == 32) {
            if (SMEM) *reinterpret_cast<uint32_t*>(sdst) = o.sc[0];
            else st_b32(sdst, o.sc[0]);
        } else {
            if (SMEM) *reinterpret_cast<uint2*>(sdst) = make_uint2(o.sc[0], o.sc[1]);
            else st_b64(sdst, make_uint2(o.sc[0], o.sc[1]));
        }
    } else {
        // zero padding [concatCol, kvCacheCol)
        int p = a.concat;
        if (SMEM || aligned) {
            for (; p < a.col && (p & 15) != 0; ++p) row[p] = 0;
            for (; p + 16 <= a.col; p += 16) *reinterpret_cast<uint4*>(row + p) = make_uint4(0u, 0u, 0u, 0u);
        }
        for (; p < a.col; ++p) row[p] = 0;
    }
}

// Shared memory: barriers (full[S], empty[S], out_free), row pointers
// [S][32], S input stages of 32 rows (pitch nseg*128 + 16), and -- with bulk
// stores -- one output buffer of 32 packed rows (pitch odd*16 bytes).
__host__ __device__ inline uint32_t ct_out_pitch(int col) { return (uint32_t)(((col + 15) / 16) | 1) * 16u; }

// S: the number of input stages (a.stages holds the same value), a template
// parameter so that the ring's stage and phase arithmetic folds to constants
// (measured 3 % faster on the mode-2 row kernel than reading it at run time).
template <int MODE, int G, int S, bool F16 = false>
__global__ void __launch_bounds__(CT_MAX_THREADS, 1) compress_tma_kernel(const CompressArgs a) {
    static_assert(S == 2 || S == 3, "stages");
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(128) uint8_t smem[];
    const int NCW = a.ncw;                         // consumer warps
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + S;
    uint64_t* out_free = empty + S;
    uint8_t** rowptr = reinterpret_cast<uint8_t**>(smem + 16 * S + 8);
    uint8_t* xs = smem + ct_header_bytes(S);
    const uint32_t row_bytes = (uint32_t)a.nseg * 128u;
    const uint32_t pitch = ct_pitch(a.nseg);
    const uint32_t stage_bytes = CT_ROWS * pitch;
    uint8_t* obuf = xs + (size_t)S * stage_bytes;
    const uint32_t opitch = ct_out_pitch(a.col);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t ntiles = (a.T + CT_ROWS - 1) / CT_ROWS;

    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], NCW);
        }
        mbar_init(out_free, 1);
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == NCW) {
        // ---------------- producer ----------------
        // the slot of the next tile's row is loaded while the current stage is
        // being consumed, so a released stage is refilled at once
        auto lane_slot = [&](int64_t tile) -> int64_t {
            const int64_t r = tile * CT_ROWS + lane;
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
            const int64_t row0 = tile * CT_ROWS;
            uint8_t* p = nullptr;
            if (slot != -1) {
                if (slot_ok(slot, a.cache.num_slots)) p = slot_row(a.cache, slot);
                else raise_fault(FAULT_SLOT_RANGE);
            }
            rowptr[st * CT_ROWS + lane] = p;
            const unsigned valid = __ballot_sync(FULL_MASK, p != nullptr);
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(&full[st], (uint32_t)__popc(valid) * row_bytes);
            __syncwarp();
            if (p != nullptr)
                bulk_copy_g2s(xs + (size_t)st * stage_bytes + (size_t)lane * pitch,
                              a.x + (row0 + lane) * a.x_row_stride, row_bytes, &full[st]);
        }
        // no copy may still be in flight when the CTA exits
        if (lane == 0)
            for (int k = it > S ? it - S : 0; k < it; ++k) mbar_wait(&full[k % S], (uint32_t)(k / S) & 1u);
        return;
    }

    // ---------------- consumers: warp -> segment column, lane -> row ----------------
    const bool aligned = a.rows_aligned != 0;
    int it = 0;
    if (a.bulk_out) {
        // warp 0 takes the rope segment (the least work) and owns the output
        // buffer: it releases it for tile `it` (out_free phase it) once the bulk
        // engine has read tile it-1's rows, waits for every warp's rows of tile
        // it (named barrier) and issues one bulk store per row.  Warp w >= 1
        // takes nope segment w - 1.  Nobody waits for another warp's reads:
        // each warp releases an input stage as soon as it has read it.
        // Every consumer warp runs every tile and makes every barrier arrival,
        // so warp 0's bar.sync always completes; after a timed-out wait a warp
        // is "dead": it skips all further waits and writes.
        const int j = warp == 0 ? a.nseg - 1 : warp - 1;
        const bool rope = (warp == 0);
        bool dead = false;
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
            const int st = it % S;
            const uint32_t round = (uint32_t)(it / S);
            if (!dead) dead = !__all_sync(FULL_MASK, mbar_wait(&full[st], round & 1u));
            uint8_t* row = dead ? nullptr : rowptr[st * CT_ROWS + lane];
            const uint8_t* xrow = xs + (size_t)st * stage_bytes + (size_t)lane * pitch;
            uint8_t* orow = obuf + (size_t)lane * opitch;
            SegOut o;
            if (row != nullptr) {
                if (!rope) ct_compute_nope<MODE, G, F16>(xrow + j * 128, o);
                else if (MODE == 2) ct_compute_rope2(a, xrow + j * 128, o);
            }
            if (rope) {
                if (it > 0) bulk_wait_read_all();    // tile it-1's rows have left the buffer
                __syncwarp();
                if (lane == 0) mbar_arrive(out_free);
            } else {
                __syncwarp();
                if (lane == 0 && !dead) mbar_arrive(&empty[st]);   // inputs read
                if (!dead) dead = !__all_sync(FULL_MASK, mbar_wait(out_free, (uint32_t)it & 1u));
                if (dead) row = nullptr;
            }
            if (row != nullptr) {
                ct_write<MODE, G, true>(a, orow, j, rope, o, xrow + j * 128, true);
                fence_proxy_async_smem();
            }
            if (rope) {
                __syncwarp();
                if (lane == 0 && !dead) mbar_arrive(&empty[st]);   // the bf16 rope was copied
                named_barrier_sync(NCW * 32);                     // every packed row is complete
                if (row != nullptr) bulk_copy_s2g(row, orow, (uint32_t)a.col);
                bulk_commit();
            } else {
                named_barrier_arrive(NCW * 32);
            }
        }
        if (warp == 0) bulk_wait_all();            // every bulk store is complete before the CTA exits
        return;
    }
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
        const int st = it % S;
        const uint32_t round = (uint32_t)(it / S);
        if (!__all_sync(FULL_MASK, mbar_wait(&full[st], round & 1u))) break;   // every lane acquires the stage
        uint8_t* row = rowptr[st * CT_ROWS + lane];
        const uint8_t* xrow = xs + (size_t)st * stage_bytes + (size_t)lane * pitch;
        if (row != nullptr) {
            for (int j = warp; j < a.nseg; j += NCW) {
                const bool rope = (j == a.nseg - 1);
                SegOut o;
                if (!rope) ct_compute_nope<MODE, G, F16>(xrow + j * 128, o);
                else if (MODE == 2) ct_compute_rope2(a, xrow + j * 128, o);
                ct_write<MODE, G, false>(a, row, j, rope, o, xrow + j * 128, aligned);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }
}

}  // namespace kvq
