// kvq_device.cuh -- device helpers shared by the epilogue kernels (sm_100a).
//
// Number formats use the hardware conversions: cvt.rn.satfinite.{e4m3x2,
// e5m2x2,e2m1x2}.f32 (round to nearest even, saturate to the largest finite
// value), cvt.rn.bf16.f32 / cvt.rn.f16.f32, cvt.rni.s32.f32.  binary32
// arithmetic uses the explicitly rounded intrinsics (__fdiv_rn, __fmul_rn,
// __fadd_rn, __fsqrt_rn) and the library is compiled with -fmad=false, so
// no multiply-add is contracted and every expression is evaluated in the
// order written.  Subnormals are kept (no -ftz).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace kvq {

constexpr unsigned FULL_MASK = 0xffffffffu;

// ---------------------------------------------------------------------------
// Device fault word: data faults (a bad slot) set bits here; the host reads
// and clears it with kvq_get_error.  One word per device (module global).
// ---------------------------------------------------------------------------
__device__ unsigned int g_fault_word;
constexpr unsigned FAULT_SLOT_RANGE = 0x1u;

__device__ __forceinline__ void raise_fault(unsigned bits) { atomicOr(&g_fault_word, bits); }

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  The library launches its kernels so that a
// kernel may be scheduled while the previous kernel of the stream is still
// finishing; every kernel calls pdl_wait() before its first global-memory
// access (reads and writes: the previous kernel may still read what this one
// overwrites), which returns once the previous kernel has completed and its
// writes are visible (at once for a kernel launched without the attribute),
// and then pdl_trigger(), which lets the next kernel's CTAs start as soon as
// this grid's CTAs leave room for them.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// 16-bit float widening (exact) and narrowing (round to nearest even)
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float f16_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu))); }
__device__ __forceinline__ float f16_hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }

// acc + x*x over the eight 16-bit values of v in index order (value 2i in the
// low half of word i), each step one multiply-add on the 16-bit operands
// (fma.rn.f32.{bf16,f16}: the operands widen exactly and the sum is rounded
// once).  That equals the separately rounded RN(acc + RN(x*x)) whenever x*x
// is exact in binary32: for every f16 value (11 significant bits, |x*x| in
// [2^-48, 2^32]), and for a bf16 value that is zero or has |x| >= 2^-67
// (8 significant bits, lowest bit >= 2^-74, so x*x is a multiple of 2^-148
// below 2^128; a square at or above 2^128 is infinite either way).
template <bool F16>
__device__ __forceinline__ float sq_acc8(const uint4& v, float acc) {
#define KVQ_SQ_ACC8(T)                                                          \
    asm("{\n\t.reg .b16 l0, h0, l1, h1, l2, h2, l3, h3;\n\t"                     \
        "mov.b32 {l0, h0}, %1;\n\tmov.b32 {l1, h1}, %2;\n\t"                     \
        "mov.b32 {l2, h2}, %3;\n\tmov.b32 {l3, h3}, %4;\n\t"                     \
        "fma.rn.f32." T " %0, l0, l0, %0;\n\tfma.rn.f32." T " %0, h0, h0, %0;\n\t" \
        "fma.rn.f32." T " %0, l1, l1, %0;\n\tfma.rn.f32." T " %0, h1, h1, %0;\n\t" \
        "fma.rn.f32." T " %0, l2, l2, %0;\n\tfma.rn.f32." T " %0, h2, h2, %0;\n\t" \
        "fma.rn.f32." T " %0, l3, l3, %0;\n\tfma.rn.f32." T " %0, h3, h3, %0;\n\t}" \
        : "+f"(acc)                                                             \
        : "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w))
    if (F16) KVQ_SQ_ACC8("f16");
    else KVQ_SQ_ACC8("bf16");
#undef KVQ_SQ_ACC8
    return acc;
}

template <bool F16>
__device__ __forceinline__ void widen8(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = F16 ? f16_lo(w[i]) : bf16_lo(w[i]);
        f[2 * i + 1] = F16 ? f16_hi(w[i]) : bf16_hi(w[i]);
    }
}

__device__ __forceinline__ uint32_t to_bf16_bits(float f) {
    unsigned short r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
    return r;
}

__device__ __forceinline__ uint32_t to_f16_bits(float f) {
    unsigned short r;
    asm("cvt.rn.f16.f32 %0, %1;" : "=h"(r) : "f"(f));
    return r;
}

// ---------------------------------------------------------------------------
// FP8 / FP4 codes.  The x2 conversions put their FIRST source operand in the
// HIGH half of the result, so (hi, lo) are passed in that order and the
// element with the lower index lands in the lower byte / nibble.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t e5m2x2(float lo, float hi) {
    unsigned short r;
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

template <bool E5M2>
__device__ __forceinline__ uint32_t fp8x2(float lo, float hi) {
    return E5M2 ? e5m2x2(lo, hi) : e4m3x2(lo, hi);
}

// Eight E2M1 codes packed into 32 bits, element 0 in bits [3:0].
__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8]) {
    uint32_t r;
    asm("{\n\t"
        ".reg .b8 q0, q1, q2, q3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
        "mov.b32 %0, {q0, q1, q2, q3};\n\t"
        "}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// Eight FP8 codes packed into two 32-bit words, element 0 in byte 0.
template <bool E5M2>
__device__ __forceinline__ uint2 fp8x8(const float (&v)[8]) {
    uint2 r;
    r.x = fp8x2<E5M2>(v[0], v[1]) | (fp8x2<E5M2>(v[2], v[3]) << 16);
    r.y = fp8x2<E5M2>(v[4], v[5]) | (fp8x2<E5M2>(v[6], v[7]) << 16);
    return r;
}

// ---------------------------------------------------------------------------
// E8M0 scale rounded up: the smallest b in [0, 254] with 2^(b-127) >= q, for a
// finite q >= 0, read off the binary32 fields of q.  A normal q = 2^(E-127) *
// 1.M needs b = E when M == 0 and E + 1 otherwise; a subnormal q < 2^-126
// needs b = 0 when q <= 2^-127 (fraction <= 2^22) and b = 1 otherwise.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e8m0_ceil(float q) {
    const uint32_t u = __float_as_uint(q) & 0x7fffffffu;
    const uint32_t E = u >> 23, M = u & 0x7fffffu;
    uint32_t b = (E == 0) ? (M > 0x400000u ? 1u : 0u) : E + (M != 0 ? 1u : 0u);
    return b > 254u ? 254u : b;
}

// 2^(127-b) as binary32 (exact; 2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float e8m0_reciprocal(uint32_t b) {
    const int k = 127 - (int)b;
    return k >= -126 ? __uint_as_float((uint32_t)(k + 127) << 23) : __uint_as_float(0x00400000u);
}

// ---------------------------------------------------------------------------
// Division by a per-group scale.  With r = RN(1/s) (one IEEE reciprocal per
// group), Markstein's correction -- P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990 -- refines q0 = RN(a r): the residual a - s q0 is exact under a fused
// multiply-add, and q = RN(q0 + residual * r).  The two-step variant repeats
// the correction once.  The quotient of a positive scale carries the sign of
// a, which also fixes the sign of a zero result.  Used only for scales with
// 2^-100 <= s < 2^101 and |a / s| <= 512, and only to produce FP8 / FP4
// codes: kvq_selftest checks, for every bf16 numerator and bf16 scale of that
// domain, that the E4M3 and E2M1 codes of the one-step quotient equal those of
// the IEEE quotient (they do, for every pair; the quotient bits themselves
// differ for about 0.2% of the pairs, never enough to move a code), and the
// constant-divisor form against IEEE division for every bf16 and f16 amax
// over 448, 57344 and 6 (bit-identical).
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool scale_in_fast_range(float s) {
    const uint32_t e = (__float_as_uint(s) >> 23) & 0xffu;
    return e >= 27u && e <= 227u;
}

__device__ __forceinline__ float with_sign_of(float q, float a) {
    return __uint_as_float(__float_as_uint(q) | (__float_as_uint(a) & 0x80000000u));
}

__device__ __forceinline__ float div_scale1(float a, float s, float r) {
    const float q0 = __fmul_rn(a, r);
    const float rem = __fmaf_rn(-q0, s, a);
    return with_sign_of(__fmaf_rn(rem, r, q0), a);
}

__device__ __forceinline__ float div_scale2(float a, float s, float r) {
    const float q0 = __fmul_rn(a, r);
    const float rem0 = __fmaf_rn(-q0, s, a);
    const float q1 = __fmaf_rn(rem0, r, q0);
    const float rem1 = __fmaf_rn(-q1, s, a);
    return with_sign_of(__fmaf_rn(rem1, r, q1), a);
}

// div_scale1 on two numerators at once with the packed binary32 pipe
// (mul.rn.f32x2 / fma.rn.f32x2: each half is the same RN operation as the
// scalar form, so the results are bit-identical to div_scale1).
__device__ __forceinline__ void div_scale1_x2(float a0, float a1, float s, float r, float& q0, float& q1) {
    asm("{\n\t.reg .b64 a, q, rem, rr, ns;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 rr, {%4, %4};\n\t"
        "mov.b64 ns, {%5, %5};\n\t"
        "mul.rn.f32x2 q, a, rr;\n\t"
        "fma.rn.f32x2 rem, q, ns, a;\n\t"
        "fma.rn.f32x2 q, rem, rr, q;\n\t"
        "mov.b64 {%0, %1}, q;\n\t}"
        : "=f"(q0), "=f"(q1)
        : "f"(a0), "f"(a1), "f"(r), "f"(-s));
    q0 = with_sign_of(q0, a0);
    q1 = with_sign_of(q1, a1);
}

// The same one-step quotient, negated, on a pair: nq = RN(a * -r) = -q0,
// rem = RN(a + s nq) = a - s q0 (exact under the fused operation), and
// t = RN(rem * -r + nq) = -RN(q0 + rem r).  t is exactly -(div_scale1(a)),
// signed zeros included (a zero numerator gives t = -0 for a = +0 and +0 for
// a = -0), so the sign fix of div_scale1 is not needed: callers encode t and
// flip the code's sign bit, which for the symmetric round-to-nearest-even,
// saturating FP8 / FP4 encodings equals encoding -t.
__device__ __forceinline__ void div_scale1_neg_x2(float a0, float a1, float s, float r, float& t0, float& t1) {
    asm("{\n\t.reg .b64 a, nq, rem, nr, ss;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 nr, {%4, %4};\n\t"
        "mov.b64 ss, {%5, %5};\n\t"
        "mul.rn.f32x2 nq, a, nr;\n\t"
        "fma.rn.f32x2 rem, nq, ss, a;\n\t"
        "fma.rn.f32x2 nq, rem, nr, nq;\n\t"
        "mov.b64 {%0, %1}, nq;\n\t}"
        : "=f"(t0), "=f"(t1)
        : "f"(a0), "f"(a1), "f"(-r), "f"(s));
}

// ---------------------------------------------------------------------------
// Packed binary32 pairs (mul/add/fma .rn.f32x2: each half is exactly the IEEE
// round-to-nearest-even scalar operation, subnormals kept).  The compiler may
// fuse a packed multiply into a following packed add, so a packed product is
// only ever fed to the addend of a fused multiply-add here, never to an add:
// plain products-then-sums stay on the scalar __fmul_rn / __fadd_rn.
// ---------------------------------------------------------------------------
// The quotient a / s of a pair by the two-step Markstein form with r = RN(1/s)
// (P. Markstein, IBM J. Res. Dev. 34(1), 1990): q0 = RN(a r); each step forms
// the exact residual a - s q under a fused multiply-add and sets
// q = RN(q + residual r).  After the first step q is faithful, so the second
// returns the correctly rounded quotient RN(a / s) whenever a, s, r and the
// quotient stay inside the normal range (the caller's guard); then the
// offset is added: (q0 + f0, q1 + f1).
__device__ __forceinline__ void div2_add_x2(float a0, float a1, float s0, float s1, float r0, float r1, float f0,
                                            float f1, float& y0, float& y1) {
    asm("{\n\t.reg .b64 a, ns, r, f, q, e;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 ns, {%4, %5};\n\t"
        "mov.b64 r, {%6, %7};\n\t"
        "mov.b64 f, {%8, %9};\n\t"
        "mul.rn.f32x2 q, a, r;\n\t"
        "fma.rn.f32x2 e, q, ns, a;\n\t"
        "fma.rn.f32x2 q, e, r, q;\n\t"
        "fma.rn.f32x2 e, q, ns, a;\n\t"
        "fma.rn.f32x2 q, e, r, q;\n\t"
        "add.rn.f32x2 q, q, f;\n\t"
        "mov.b64 {%0, %1}, q;\n\t}"
        : "=f"(y0), "=f"(y1)
        : "f"(a0), "f"(a1), "f"(-s0), "f"(-s1), "f"(r0), "f"(r1), "f"(f0), "f"(f1));
}

// The two-step quotient of div2_add_x2 without the offset, one common divisor
// s with r = RN(1/s), signed zeros kept (a zero numerator gives a zero of its
// sign): (RN(a0 / s), RN(a1 / s)) under the same range conditions.
__device__ __forceinline__ void div2_x2(float a0, float a1, float s, float r, float& q0, float& q1) {
    asm("{\n\t.reg .b64 a, ns, rr, q, e;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 ns, {%4, %4};\n\t"
        "mov.b64 rr, {%5, %5};\n\t"
        "mul.rn.f32x2 q, a, rr;\n\t"
        "fma.rn.f32x2 e, q, ns, a;\n\t"
        "fma.rn.f32x2 q, e, rr, q;\n\t"
        "fma.rn.f32x2 e, q, ns, a;\n\t"
        "fma.rn.f32x2 q, e, rr, q;\n\t"
        "mov.b64 {%0, %1}, q;\n\t}"
        : "=f"(q0), "=f"(q1)
        : "f"(a0), "f"(a1), "f"(-s), "f"(r));
    q0 = with_sign_of(q0, a0);
    q1 = with_sign_of(q1, a1);
}

// (a0 b0, a1 b1), each product rounded once (mul.rn.f32x2: each half is the
// IEEE round-to-nearest-even product).  Used only where the products feed
// another multiply or a conversion, never an add (no contraction can arise).
__device__ __forceinline__ void mul_x2(float a0, float a1, float b0, float b1, float& r0, float& r1) {
    asm("{\n\t.reg .b64 a, b, r;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 b, {%4, %5};\n\t"
        "mul.rn.f32x2 r, a, b;\n\t"
        "mov.b64 {%0, %1}, r;\n\t}"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// a / s for nonzero numerators of at most 11 significant bits (bf16 or f16
// values) by one correction step: q0 = RN(a r), e = a - q0 s (formed exactly
// by the fused operation), q = RN(q0 + e r), with r = RN(1/s).  It equals
// IEEE division whenever the reciprocal, the quotient and the residual stay
// normal binary32 numbers: kvq_selftest 10 runs every bf16 and f16
// numerator mantissa against every binary32 divisor mantissa, and 9 the
// rmsnorm kernels' guard domain (their bounds on rms and |x| keep the three
// normal).
__device__ __forceinline__ void div1_x2_nz(float a0, float a1, float s, float r, float& q0, float& q1) {
    asm("{\n\t.reg .b64 a, ns, rr, q, e;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 ns, {%4, %4};\n\t"
        "mov.b64 rr, {%5, %5};\n\t"
        "mul.rn.f32x2 q, a, rr;\n\t"
        "fma.rn.f32x2 e, q, ns, a;\n\t"
        "fma.rn.f32x2 q, e, rr, q;\n\t"
        "mov.b64 {%0, %1}, q;\n\t}"
        : "=f"(q0), "=f"(q1)
        : "f"(a0), "f"(a1), "f"(-s), "f"(r));
}

// Two binary32 values rounded to bf16 (F16: f16), lo in bits [15:0].
template <bool F16>
__device__ __forceinline__ uint32_t half2_bits(float lo, float hi) {
    uint32_t r;
    if (F16) asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    else asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Eight FP8 codes (E4M3, or E5M2), element 0 in bits [7:0].
template <bool E5M2>
__device__ __forceinline__ uint2 fp8x8_packed(const float (&v)[8]) {
    uint2 r;
    if (E5M2)
        asm("{\n\t.reg .b16 c0, c1, c2, c3;\n\t"
            "cvt.rn.satfinite.e5m2x2.f32 c0, %3, %2;\n\t"
            "cvt.rn.satfinite.e5m2x2.f32 c1, %5, %4;\n\t"
            "cvt.rn.satfinite.e5m2x2.f32 c2, %7, %6;\n\t"
            "cvt.rn.satfinite.e5m2x2.f32 c3, %9, %8;\n\t"
            "mov.b32 %0, {c0, c1};\n\tmov.b32 %1, {c2, c3};\n\t}"
            : "=r"(r.x), "=r"(r.y)
            : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    else
        asm("{\n\t.reg .b16 c0, c1, c2, c3;\n\t"
            "cvt.rn.satfinite.e4m3x2.f32 c0, %3, %2;\n\t"
            "cvt.rn.satfinite.e4m3x2.f32 c1, %5, %4;\n\t"
            "cvt.rn.satfinite.e4m3x2.f32 c2, %7, %6;\n\t"
            "cvt.rn.satfinite.e4m3x2.f32 c3, %9, %8;\n\t"
            "mov.b32 %0, {c0, c1};\n\tmov.b32 %1, {c2, c3};\n\t}"
            : "=r"(r.x), "=r"(r.y)
            : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// Four binary32 values rounded half to even to integers and saturated to
// int8, packed little-endian (value 0 in byte 0).  NaN gives 0.
__device__ __forceinline__ uint32_t int8x4_rne_sat(float v0, float v1, float v2, float v3) {
    int32_t i0, i1, i2, i3;
    asm("cvt.rni.s32.f32 %0, %1;" : "=r"(i0) : "f"(v0));
    asm("cvt.rni.s32.f32 %0, %1;" : "=r"(i1) : "f"(v1));
    asm("cvt.rni.s32.f32 %0, %1;" : "=r"(i2) : "f"(v2));
    asm("cvt.rni.s32.f32 %0, %1;" : "=r"(i3) : "f"(v3));
    uint32_t hi, r;
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, 0;" : "=r"(hi) : "r"(i3), "r"(i2));
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(i1), "r"(i0), "r"(hi));
    return r;
}

// Static int8 of four values: round half to even of o / scale + offset,
// saturated (offset 0 when absent), packed little-endian.  r holds RN(1/scale)
// for channels whose scale lies in [2^-60, 2^60] and whose |offset| <= 2^16,
// else 0.  When every r is set and every |o| <= 2^60 the quotient comes
// from the two-step Markstein form, which is then exact wherever the result
// depends on it: a quotient in [2^-30, 2^20] has normal operands, residuals
// and result, so it equals the IEEE quotient; below 2^-30 the rounded sum
// with any binary32 offset, hence the integer, does not depend on the
// quotient's last bits; above 2^20 the integer saturates either way.  Other
// lanes divide with IEEE division.  kvq_selftest 6 checks the two paths
// against each other on random and near-tie triples.  The quotients run on
// packed pairs (div2_add_x2).
__device__ __forceinline__ uint32_t int8x4_quant(const float (&o)[4], const float (&s)[4], const float (&f)[4],
                                                 const float (&r)[4]) {
    float q[4];
    const float m = fmaxf(fmaxf(fabsf(o[0]), fabsf(o[1])), fmaxf(fabsf(o[2]), fabsf(o[3])));
    const float rmin = fminf(fminf(r[0], r[1]), fminf(r[2], r[3]));
    if (m <= 1.152921504606846976e18f && rmin > 0.0f) {      // |o| <= 2^60, every channel eligible
        div2_add_x2(o[0], o[1], s[0], s[1], r[0], r[1], f[0], f[1], q[0], q[1]);
        div2_add_x2(o[2], o[3], s[2], s[3], r[2], r[3], f[2], f[3], q[2], q[3]);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = __fadd_rn(__fdiv_rn(o[k], s[k]), f[k]);
    }
    return int8x4_rne_sat(q[0], q[1], q[2], q[3]);
}

// RN(1/scale) where the fast quotient of int8x4_quant applies, else 0
__device__ __forceinline__ float int8_quant_rcp(float sc, float of) {
    const uint32_t e = (__float_as_uint(sc) >> 23) & 0xffu;
    const bool ok = sc > 0.0f && e >= 67u && e <= 187u && fabsf(of) <= 65536.0f;
    return ok ? __frcp_rn(sc) : 0.0f;
}

// Largest magnitude of the two bf16 halves of a and b, per half (max of the
// absolute values; the sign bits of the result are not meaningful).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Smallest magnitude of the two 16-bit halves of a and b, per half (the sign
// bits of the result are not meaningful; a NaN half yields the other
// operand's half).
template <bool F16>
__device__ __forceinline__ uint32_t absmin_x2(uint32_t a, uint32_t b) {
    uint32_t r;
    if (F16) asm("min.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    else asm("min.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// The same for two f16 halves.
__device__ __forceinline__ uint32_t absmax_f16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// The value of a 16-bit float's bit pattern (bf16 or f16)
template <bool F16>
__device__ __forceinline__ float half_value(uint32_t bits) {
    return F16 ? __half2float(__ushort_as_half((unsigned short)bits)) : __uint_as_float(bits << 16);
}

// eight quotients f[i] / s through div_scale1_x2
__device__ __forceinline__ void div_scale8(const float (&f)[8], float s, float r, float (&q)[8]) {
#pragma unroll
    for (int i = 0; i < 8; i += 2) div_scale1_x2(f[i], f[i + 1], s, r, q[i], q[i + 1]);
}

// amax / c for the format maxima c = 448, 57344, 6 (amax >= 0, a bf16 value):
// the one-step form with the constant RN(1/c).
__device__ __forceinline__ float div_by_fmax(float amax, float c) {
    // RN(1/448) = 0x3b124925, RN(1/6) = 0x3e2aaaab, RN(1/57344) = 0x37924925
    const float r = __uint_as_float(c == 448.0f ? 0x3b124925u : (c == 6.0f ? 0x3e2aaaabu : 0x37924925u));
    const float q0 = __fmul_rn(amax, r);
    const float rem = __fmaf_rn(-q0, c, amax);
    return __fmaf_rn(rem, r, q0);
}

// Static int8: round half to even, saturate to [-128, 127]; NaN -> 0.
__device__ __forceinline__ int32_t int8_rne_sat(float v) {
    int r;
    asm("cvt.rni.s32.f32 %0, %1;" : "=r"(r) : "f"(v));
    return r < -128 ? -128 : (r > 127 ? 127 : r);
}

// Largest |x| of eight 16-bit floats as the bits of one of them (for finite
// inputs the magnitude order equals the integer order of the bit patterns).
__device__ __forceinline__ uint32_t absmax_bits8(const uint4& v) {
    const uint32_t m = 0x7fff7fffu;
    uint32_t a = __vmaxu2(v.x & m, v.y & m);
    uint32_t b = __vmaxu2(v.z & m, v.w & m);
    a = __vmaxu2(a, b);
    return max(a & 0xffffu, a >> 16);
}

// ---------------------------------------------------------------------------
// Loads and stores.  Every store checks the alignment of its own address, so
// packed rows of any byte length (e.g. 323) are written correctly; aligned
// rows take the vector path.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    return __ldcs(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ void st_b8(uint8_t* p, uint32_t v) { *p = (uint8_t)v; }

__device__ __forceinline__ void st_b16(uint8_t* p, uint32_t v) {
    if ((reinterpret_cast<uintptr_t>(p) & 1) == 0) {
        *reinterpret_cast<uint16_t*>(p) = (uint16_t)v;
    } else {
        p[0] = (uint8_t)v;
        p[1] = (uint8_t)(v >> 8);
    }
}

__device__ __forceinline__ void st_b32(uint8_t* p, uint32_t v) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    if ((a & 3) == 0) {
        *reinterpret_cast<uint32_t*>(p) = v;
    } else if ((a & 1) == 0) {
        reinterpret_cast<uint16_t*>(p)[0] = (uint16_t)v;
        reinterpret_cast<uint16_t*>(p)[1] = (uint16_t)(v >> 16);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) p[k] = (uint8_t)(v >> (8 * k));
    }
}

__device__ __forceinline__ void st_b64(uint8_t* p, uint2 v) {
    if ((reinterpret_cast<uintptr_t>(p) & 7) == 0) {
        *reinterpret_cast<uint2*>(p) = v;
    } else {
        st_b32(p, v.x);
        st_b32(p + 4, v.y);
    }
}

__device__ __forceinline__ void st_b128(uint8_t* p, uint4 v) {
    if ((reinterpret_cast<uintptr_t>(p) & 15) == 0) {
        *reinterpret_cast<uint4*>(p) = v;
    } else {
        st_b64(p, make_uint2(v.x, v.y));
        st_b64(p + 8, make_uint2(v.z, v.w));
    }
}

// 32 16-bit values (64 bytes) at p as 16 words (value 2i in the low half of word i).
__device__ __forceinline__ void ld_slice(const uint16_t* p, int vec, uint32_t (&w)[16]) {
    if (vec == 2) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
            asm("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                : "=r"(w[8 * h]), "=r"(w[8 * h + 1]), "=r"(w[8 * h + 2]), "=r"(w[8 * h + 3]), "=r"(w[8 * h + 4]),
                  "=r"(w[8 * h + 5]), "=r"(w[8 * h + 6]), "=r"(w[8 * h + 7])
                : "l"(p + 16 * h));
    } else if (vec == 1) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint4 v = ld_stream16(p + 8 * k);
            w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = (uint32_t)__ldcs(p + 2 * i) | ((uint32_t)__ldcs(p + 2 * i + 1) << 16);
    }
}

// 32 bytes at p (8 words, little-endian).
__device__ __forceinline__ void st_32B(uint8_t* p, const uint32_t* w, bool vec32) {
    if (vec32) {
        asm volatile("st.global.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]),
                     "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                     : "memory");
    } else {
        st_b128(p, make_uint4(w[0], w[1], w[2], w[3]));
        st_b128(p + 16, make_uint4(w[4], w[5], w[6], w[7]));
    }
}

// |x| maximum (as bf16 bits) of the 2*N values in words w[i0 .. i0+N)
template <int N>
__device__ __forceinline__ uint32_t absmax_words(const uint32_t (&w)[16], int i0) {
    const uint32_t msk = 0x7fff7fffu;
    uint32_t m = w[i0] & msk;
#pragma unroll
    for (int i = 1; i < N; ++i) m = __vmaxu2(m, w[i0 + i] & msk);
    return max(m & 0xffffu, m >> 16);
}

__device__ __forceinline__ int64_t load_slot(const void* slots, int is64, int64_t i) {
    return is64 ? reinterpret_cast<const int64_t*>(slots)[i] : (int64_t) reinterpret_cast<const int32_t*>(slots)[i];
}

// ---------------------------------------------------------------------------
// Paged cache rows: slot s -> block s / block_size, row s % block_size.
// ---------------------------------------------------------------------------
struct PagedRows {
    uint8_t* base;
    int64_t num_slots;
    int64_t block_size;
    int64_t row_bytes;
    int64_t block_stride;  // bytes
    int32_t bs_shift;      // log2(block_size) when block_size is a power of two, else -1
};

__device__ __forceinline__ uint8_t* slot_row(const PagedRows& c, int64_t s) {
    if (c.bs_shift >= 0) {
        const int64_t blk = s >> c.bs_shift;
        return c.base + blk * c.block_stride + (s & (c.block_size - 1)) * c.row_bytes;
    }
    if (c.num_slots <= 0x7fffffff) {
        const uint32_t us = (uint32_t)s, bs = (uint32_t)c.block_size;
        const uint32_t blk = us / bs;
        return c.base + (int64_t)blk * c.block_stride + (int64_t)(us - blk * bs) * c.row_bytes;
    }
    const int64_t blk = s / c.block_size;
    return c.base + blk * c.block_stride + (s - blk * c.block_size) * c.row_bytes;
}

// -1 -> skip silently; other values outside [0, num_slots) -> skip and flag.
__device__ __forceinline__ bool slot_ok(int64_t s, int64_t num_slots) {
    return s >= 0 && s < num_slots;
}

}  // namespace kvq
