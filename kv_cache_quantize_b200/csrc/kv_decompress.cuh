// kv_decompress.cuh -- packed-row decoder: the inverse of kv_compress_epilog
// (aclnnKvCompressEpilog, 计算公式 scenarios 1-3 and the row layout of its
// 约束说明, read backwards: code value x stored group scale, one rounding to
// bf16 -- or to f16 in modes 0/1 for rows written from f16 x; the 16-bit rope
// of modes 0/1 is copied, the FP8 rope of mode 2 is divided by xScale).
//
// Work decomposition.  A row of d values is d/32 SLICES of 32 values: the
// nn = (d-64)/32 nope slices (nn is even), then the two rope slices.  One
// lane owns one slice: it reads the slice's codes (32 bytes FP8 or 16 bytes
// FP4) and its group's scale from the packed row, and writes the slice's 64
// bytes of 16-bit output.  A warp takes a CHUNK of 32 slices:
//   modes 0/1: 32 consecutive slices of the flattened [T, d/32] slice array,
//     so a warp's stores cover one contiguous stretch of y (the rope is a
//     plain copy, as cheap as a nope slice);
//   mode 2: rows in blocks of 16, whose 16 nn nope slices form nn/2 chunks
//     (row-major) and whose 32 rope slices one more chunk, so every chunk is
//     all nope or all rope and the decode path is uniform across the warp
//     (the rope's table lookups and the FP4 path would otherwise run one
//     after the other in every warp that holds both).
// Grid-stride over the chunks, software-pipelined: the slots of chunk i+2 and
// the packed bytes of chunk i+1 are in flight while chunk i is decoded.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

constexpr int DC_THREADS = 256;

struct DecompressArgs {
    PagedRows cache;
    const void* slots;      // int32 or int64
    int32_t slots_i64;
    int64_t T;
    uint16_t* y;            // bf16 (or f16, modes 0/1) [T, d], row stride y_row_stride elements
    int64_t y_row_stride;
    int32_t nslice;         // d / 32
    int32_t n;              // d - 64
    float x_scale;          // mode 2 rope divisor
    int32_t rows_vec16;     // every packed row starts on a 16-byte boundary
    int32_t y_vec32;        // y rows start on 32-byte boundaries
};

// NB (16, 32 or 64) packed bytes at p into words, whatever p's alignment
template <int NB>
__device__ __forceinline__ void dc_load(const uint8_t* p, bool vec16, uint32_t (&w)[16]) {
    if (vec16) {
#pragma unroll
        for (int k = 0; k < NB / 16; ++k) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(p + 16 * k));
            w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < NB / 4; ++k)
            w[k] = (uint32_t)__ldg(p + 4 * k) | ((uint32_t)__ldg(p + 4 * k + 1) << 8) |
                   ((uint32_t)__ldg(p + 4 * k + 2) << 16) | ((uint32_t)__ldg(p + 4 * k + 3) << 24);
    }
}

__device__ __forceinline__ uint32_t dc_ld16(const uint8_t* p) {
    return (uint32_t)__ldg(p) | ((uint32_t)__ldg(p + 1) << 8);
}

// two FP8 E4M3 codes (low byte first) -> their values (exact, through f16)
__device__ __forceinline__ void e4m3x2_to_f32(uint32_t c2, float& lo, float& hi) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((unsigned short)c2));
    lo = f16_lo(h);
    hi = f16_hi(h);
}

// two FP4 E2M1 codes (even element in the low nibble) -> their values
__device__ __forceinline__ void e2m1x2_to_f32(uint32_t c2, float& lo, float& hi) {
    uint32_t h;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u16 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(h)
        : "h"((unsigned short)(c2 & 0xffu)));
    lo = f16_lo(h);
    hi = f16_hi(h);
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t f16x2_rn(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// the output pair in y's dtype (YF16: f16, modes 0/1 only; else bf16)
template <bool YF16>
__device__ __forceinline__ uint32_t out_x2(float lo, float hi) {
    return YF16 ? f16x2_rn(lo, hi) : bf16x2_rn(lo, hi);
}

// 2^(b-127) for an E8M0 byte b (b = 0: the subnormal 2^-127; b = 255: inf)
__device__ __forceinline__ float e8m0_value(uint32_t b) {
    return b == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(b << 23);
}

// one slice of a live row: decode w (codes, or the stored rope) with scale bits sc
// rope_tab (mode 2): bf16_rn(E4M3 value / xScale) for each of the 256 codes
template <int MODE, int G, bool YF16>
__device__ __forceinline__ void dc_slice(const DecompressArgs& a, int nn, const uint32_t (&w)[16], uint32_t sc,
                                         int j, uint16_t* yrow, const uint16_t* rope_tab) {
    uint32_t out[16];
    if (j >= nn) {
        if (MODE != 2) {
            // the bf16 rope, copied
#pragma unroll
            for (int k = 0; k < 16; ++k) out[k] = w[k];
        } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint32_t c2 = w[k >> 1] >> (16 * (k & 1));
                out[k] = (uint32_t)rope_tab[c2 & 0xffu] | ((uint32_t)rope_tab[(c2 >> 8) & 0xffu] << 16);
            }
        }
    } else if (MODE == 0 || MODE == 1) {
        const float sf = MODE == 0 ? __uint_as_float(sc << 16) : e8m0_value(sc);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            float lo, hi;
            e4m3x2_to_f32(w[k >> 1] >> (16 * (k & 1)), lo, hi);
            out[k] = out_x2<YF16>(__fmul_rn(lo, sf), __fmul_rn(hi, sf));
        }
    } else {
        // 16 bytes of FP4 codes; G = 16: two scales (sc low half first), else one
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float sf = __uint_as_float((G == 16 ? (k < 8 ? sc & 0xffffu : sc >> 16) : sc & 0xffffu) << 16);
            float lo, hi;
            e2m1x2_to_f32(w[k >> 2] >> (8 * (k & 3)), lo, hi);
            out[k] = bf16x2_rn(__fmul_rn(lo, sf), __fmul_rn(hi, sf));
        }
    }
    uint8_t* yp = reinterpret_cast<uint8_t*>(yrow + 32 * j);
    st_32B(yp, out, a.y_vec32 != 0);
    st_32B(yp + 32, out + 8, a.y_vec32 != 0);
}

// packed bytes a slice needs: its codes (or the 64 bytes of a bf16 rope) in w,
// its group scale bits in sc (nn: the number of nope slices)
template <int MODE, int G, bool DBL>
__device__ __forceinline__ void dc_fetch(const DecompressArgs& a, int nn, const uint8_t* row, int j,
                                         uint32_t (&w)[16], uint32_t& sc) {
    const bool v16 = a.rows_vec16 != 0;
    sc = 0u;
    if (DBL && j < nn) {
        // mode 2, G = 32 or 64: the two nope slices j, j + 1 (j even): 32 code bytes
        // and their scale(s), the slice-j scale in the low half
        dc_load<32>(row + 16 * j, v16, w);
        const uint8_t* sp = row + a.n / 2 + 64;
        sc = G == 32 ? (dc_ld16(sp + 2 * j) | (dc_ld16(sp + 2 * j + 2) << 16)) : dc_ld16(sp + 2 * (j >> 1));
        return;
    }
    if (j >= nn) {
        if (MODE != 2) dc_load<64>(row + a.n + 64 * (j - nn), v16, w);
        else dc_load<32>(row + a.n / 2 + 32 * (j - nn), v16, w);
        return;
    }
    if (MODE == 2) {
        dc_load<16>(row + 16 * j, v16, w);
        const uint8_t* sp = row + a.n / 2 + 64;
        if (G == 16) sc = dc_ld16(sp + 4 * j) | (dc_ld16(sp + 4 * j + 2) << 16);
        else if (G == 32) sc = dc_ld16(sp + 2 * j);
        else sc = dc_ld16(sp + 2 * (j >> 1));
    } else {
        dc_load<32>(row + 32 * j, v16, w);
        sc = MODE == 0 ? dc_ld16(row + a.n + 128 + 2 * (j >> 1)) : (uint32_t)__ldg(row + a.n + 128 + (j >> 1));
    }
}

__device__ __forceinline__ int64_t dc_slot(const DecompressArgs& a, int64_t row, bool act) {
    if (!act) return -1;
    return a.slots_i64 ? reinterpret_cast<const int64_t*>(a.slots)[row]
                       : (int64_t) reinterpret_cast<const int32_t*>(a.slots)[row];
}

// Row of a slot (nullptr: skipped or out of range; the slice-0 lane of the
// token raises the fault for an out-of-range slot).
__device__ __forceinline__ const uint8_t* dc_row(const DecompressArgs& a, int64_t s, int j) {
    if (s == -1) return nullptr;
    if (!slot_ok(s, a.cache.num_slots)) {
        if (j == 0) raise_fault(FAULT_SLOT_RANGE);
        return nullptr;
    }
    return slot_row(a.cache, s);
}

// NS: slices per row (d / 32) when known at compile time (18: d = 576), else 0
// and a.nslice; the constant form measured 11 % faster in mode 0 at d = 576.
// DBL (mode 2, G = 32 or 64, (d - 64) / 32 a multiple of 4): a nope lane takes
// two adjacent slices (32 bytes of FP4 codes, as many as a mode-0 slice), so a
// 16-row block is (d - 64) / 128 nope chunks and one rope chunk.
template <int MODE, int G, int NS, bool YF16 = false, bool DBL = false>
__global__ void __launch_bounds__(DC_THREADS, (NS != 0 || (MODE == 2 && !DBL)) ? 4 : 3) kv_decompress_kernel(const DecompressArgs a) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int ns = NS ? NS : a.nslice;
    const int nn = ns - 2;
    const int hn = DBL ? nn / 4 : nn / 2;       // mode 2: nope chunks per block of 16 rows
    const int64_t nchunks = MODE == 2 ? ((a.T + 15) / 16) * (hn + 1) : (a.T * ns + 31) / 32;
    // mode 2: the decoded rope value of every E4M3 code, one IEEE division each
    __shared__ uint16_t rope_tab[MODE == 2 ? 256 : 1];
    if (MODE == 2) {
        for (int c = threadIdx.x; c < 256; c += blockDim.x) {
            float lo, hi;
            e4m3x2_to_f32((uint32_t)c, lo, hi);
            rope_tab[c] = (uint16_t)(bf16x2_rn(__fdiv_rn(lo, a.x_scale), 0.0f) & 0xffffu);
        }
        __syncthreads();
    }
    if (gwarp >= nchunks) return;
    // the lane's slice (row, j) in chunk c: modes 0/1 step through the flat
    // slice array (chunk c + nwarps is nwarps * 32 slices further, added
    // without a division); mode 2 locates it in its 16-row block
    const int64_t step = nwarps * 32;
    const int64_t qs = step / ns;
    const int rs = (int)(step - qs * ns);
    auto advance = [&](int64_t& r, int& j) {
        r += qs;
        j += rs;
        if (j >= ns) {
            j -= ns;
            ++r;
        }
    };
    auto locate = [&](int64_t c, int64_t& r, int& j) {
        const int64_t blk = c / (hn + 1);
        const int w = (int)(c - blk * (hn + 1));
        if (w < hn) {
            const int per = DBL ? nn / 2 : nn;          // lanes per row
            const int sl = 32 * w + lane;
            r = 16 * blk + sl / per;
            j = (sl - (sl / per) * per) * (DBL ? 2 : 1);
        } else {
            r = 16 * blk + (lane >> 1);
            j = nn + (lane & 1);
        }
    };
    int64_t row0, row1;
    int j0, j1;
    if (MODE == 2) {
        locate(gwarp, row0, j0);
        locate(gwarp + nwarps, row1, j1);
    } else {
        const int64_t hs = gwarp * 32 + lane;
        row0 = hs / ns;
        j0 = (int)(hs - row0 * ns);
        row1 = row0;
        j1 = j0;
        advance(row1, j1);
    }
    const int64_t s0 = dc_slot(a, row0, row0 < a.T);
    int64_t s1 = dc_slot(a, row1, row1 < a.T && gwarp + nwarps < nchunks);
    const uint8_t* p0 = dc_row(a, s0, j0);
    uint32_t w0[16], w1[16], sc0 = 0u, sc1 = 0u;
    if (p0) dc_fetch<MODE, G, DBL>(a, nn, p0, j0, w0, sc0);
    for (int64_t c = gwarp; c < nchunks; c += nwarps) {
        int64_t row2 = row1;
        int j2 = j1;
        if (MODE == 2) locate(c + 2 * nwarps, row2, j2);
        else advance(row2, j2);
        const int64_t s2 = dc_slot(a, row2, row2 < a.T && c + 2 * nwarps < nchunks);
        const uint8_t* p1 = dc_row(a, s1, j1);
        if (p1) dc_fetch<MODE, G, DBL>(a, nn, p1, j1, w1, sc1);
        if (p0) {
            uint16_t* yrow = a.y + row0 * a.y_row_stride;
            dc_slice<MODE, G, YF16>(a, nn, w0, sc0, j0, yrow, rope_tab);
            if (DBL && j0 < nn) {
                // the second slice: codes w0[4..7], its own scale (G = 32) or the shared one
                uint32_t w2[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) w2[i] = i < 4 ? w0[4 + i] : 0u;
                dc_slice<MODE, G, YF16>(a, nn, w2, G == 32 ? sc0 >> 16 : sc0, j0 + 1, yrow, rope_tab);
            }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) w0[i] = w1[i];
        sc0 = sc1;
        p0 = p1;
        row0 = row1;
        j0 = j1;
        row1 = row2;
        j1 = j2;
        s1 = s2;
    }
}

}  // namespace kvq
