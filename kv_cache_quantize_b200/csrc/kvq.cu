// kvq.cu -- host side of the C ABI declared in include/kvq.h: argument
// validation, kernel selection and launch.  Single translation unit: the
// kernels live in the .cuh files included below.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <utility>

#include <nvtx3/nvToolsExt.h>

#include "kvq.h"
#include "compress_epilog.cuh"
#include "compressor.cuh"
#include "dequant_rope_quant.cuh"
#include "indexer_quant.cuh"
#include "kv_decompress.cuh"
#include "rmsnorm_rope.cuh"
#include "scatter_copy.cuh"

namespace {

using namespace kvq;

// ---------------------------------------------------------------------------
// descriptor helpers
// ---------------------------------------------------------------------------
int64_t elem_bytes(int32_t dt) {
    switch (dt) {
        case KVQ_BF16: case KVQ_F16: return 2;
        case KVQ_F32: case KVQ_I32: return 4;
        case KVQ_I64: return 8;
        case KVQ_I8: case KVQ_U8: case KVQ_F8E4M3: case KVQ_F8E5M2: case KVQ_E8M0: return 1;
        default: return 0;
    }
}

bool valid_desc(const kvq_tensor* t) {
    if (!t || t->ndim < 0 || t->ndim > KVQ_MAX_DIMS || elem_bytes(t->dtype) == 0) return false;
    for (int i = 0; i < t->ndim; ++i)
        if (t->shape[i] < 0) return false;
    return true;
}

int64_t numel(const kvq_tensor* t) {
    int64_t n = 1;
    for (int i = 0; i < t->ndim; ++i) n *= t->shape[i];
    return n;
}

int64_t numel_leading(const kvq_tensor* t) {
    int64_t n = 1;
    for (int i = 0; i + 1 < t->ndim; ++i) n *= t->shape[i];
    return n;
}

// Row-major contiguous (dimensions of size 1 may carry any stride).
bool contiguous(const kvq_tensor* t) {
    if (numel(t) == 0) return true;   // no elements: any strides describe it
    int64_t expect = 1;
    for (int i = t->ndim - 1; i >= 0; --i) {
        if (t->shape[i] == 1) continue;
        if (t->stride[i] != expect) return false;
        expect *= t->shape[i];
    }
    return true;
}

// Last dimension contiguous and the leading dimensions flattenable into rows
// with one row stride (in elements).
bool flatten_rows(const kvq_tensor* t, int64_t* rows, int64_t* row_stride) {
    if (t->ndim < 1) return false;
    const int64_t d = t->shape[t->ndim - 1];
    if (numel(t) == 0) {             // no elements: any strides describe it
        *rows = d == 0 ? 0 : numel_leading(t);
        *row_stride = d;
        return true;
    }
    if (d > 1 && t->stride[t->ndim - 1] != 1) return false;
    int64_t r = 1, rs = -1, expect = -1;
    for (int i = t->ndim - 2; i >= 0; --i) {
        r *= t->shape[i];
        if (t->shape[i] == 1) continue;
        if (rs < 0) {
            rs = t->stride[i];
        } else if (t->stride[i] != expect) {
            return false;
        }
        expect = t->stride[i] * t->shape[i];
    }
    if (rs < 0) rs = d;
    if (r > 1 && rs < d) return false;
    *rows = r;
    *row_stride = rs;
    return true;
}

// A cache [blockNum, a, b, headDim] with one of a/b equal to 1 (the other is
// blockSize) -- or, when inner > 1, [blockNum, blockSize, inner, headDim].
// Rows of inner*headDim elements are contiguous inside a block; only the
// block dimension may be strided.
kvq_status paged_from(const kvq_tensor* c, int64_t inner, PagedRows* out, int64_t* head_dim) {
    if (c->ndim != 4) return KVQ_ERR_NDIM;
    const int64_t eb = elem_bytes(c->dtype);
    const int64_t hd = c->shape[3];
    int64_t bs;
    int bs_dim;
    if (inner > 1) {
        if (c->shape[2] != inner) return KVQ_ERR_SHAPE;
        bs = c->shape[1];
        bs_dim = 1;
        if (hd > 1 && c->stride[3] != 1) return KVQ_ERR_LAYOUT;
        if (inner > 1 && c->stride[2] != hd) return KVQ_ERR_LAYOUT;
        if (bs > 1 && c->stride[1] != inner * hd) return KVQ_ERR_LAYOUT;
    } else {
        if (c->shape[2] == 1) { bs = c->shape[1]; bs_dim = 1; }
        else if (c->shape[1] == 1) { bs = c->shape[2]; bs_dim = 2; }
        else return KVQ_ERR_SHAPE;
        if (hd > 1 && c->stride[3] != 1) return KVQ_ERR_LAYOUT;
        if (bs > 1 && c->stride[bs_dim] != hd) return KVQ_ERR_LAYOUT;
    }
    const int64_t nb = c->shape[0];
    const int64_t row = inner * hd;
    if (nb > 1 && c->stride[0] < bs * row) return KVQ_ERR_LAYOUT;
    out->base = static_cast<uint8_t*>(c->data);
    out->num_slots = nb * bs;
    out->block_size = bs;
    out->row_bytes = row * eb;
    out->block_stride = (nb > 1 ? c->stride[0] : bs * row) * eb;
    out->bs_shift = -1;
    for (int k = 0; k < 62; ++k)
        if (bs == (int64_t(1) << k)) out->bs_shift = k;
    *head_dim = hd;
    return KVQ_OK;
}

bool is_index_dtype(int32_t dt) { return dt == KVQ_I32 || dt == KVQ_I64; }

// A named NVTX range over one C-ABI call (visible in profilers; a no-op
// unless a tool is attached).
struct Trace {
    explicit Trace(const char* name) { nvtxRangePushA(name); }
    ~Trace() { nvtxRangePop(); }
};

// ---------------------------------------------------------------------------
// launch sizing: a grid of (SMs x resident blocks) persistent blocks at most
// ---------------------------------------------------------------------------
int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

// Resident blocks per SM of a kernel at a launch shape, asked of the runtime
// once per (kernel, device, threads, shared memory) and remembered: the
// query costs host time on every call otherwise.  Kernels with dynamic shared
// memory get their opt-in limit raised to the device maximum on first use.
int resident_blocks(const void* fn, int threads, size_t smem) {
    struct Entry { const void* fn; int dev, threads; size_t smem; int occ; };
    static std::mutex mu;
    static Entry table[512];
    static int used = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (table[i].fn == fn && table[i].dev == dev && table[i].threads == threads && table[i].smem == smem)
            return table[i].occ;
    bool attr_set = false;          // the shared-memory limit was raised by an earlier entry
    for (int i = 0; i < used; ++i)
        if (table[i].fn == fn && table[i].dev == dev && table[i].smem > 0) attr_set = true;
    if (smem > 0 && !attr_set) {
        int optin = 0;
        if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || optin <= 0)
            optin = 227 * 1024;
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    }
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, threads, smem) != cudaSuccess || occ < 1) occ = 1;
    if (used < 512) table[used++] = Entry{fn, dev, threads, smem, occ};
    return occ;
}

template <typename K>
int64_t persistent_grid(K kernel, int threads, int64_t needed_blocks, size_t smem = 0) {
    const int occ = resident_blocks(reinterpret_cast<const void*>(kernel), threads, smem);
    const int64_t cap = (int64_t)sm_count() * occ;
    int64_t g = needed_blocks < cap ? needed_blocks : cap;
    return g < 1 ? 1 : g;
}

// Launch with programmatic stream serialization (see pdl_wait in
// kvq_device.cuh): the kernel may be scheduled before the previous kernel of
// the stream completes and waits for it on the device.
// Returns the launch's own status (not cudaGetLastError, which would also
// report -- and clear -- errors left by unrelated earlier CUDA work).
template <typename... P, typename... A>
cudaError_t launch(void (*kernel)(P...), unsigned grid, unsigned block, size_t smem, cudaStream_t s, A&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

kvq_status launched(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

// ---------------------------------------------------------------------------
// fault word read-and-clear (kvq_get_error): one atomic exchange on the device
// into a snapshot slot that the host then copies back
// ---------------------------------------------------------------------------
constexpr uint32_t FAULT_SNAPSHOTS = 64;
__device__ unsigned int g_fault_snapshot[FAULT_SNAPSHOTS];

__global__ void fault_exchange_kernel(uint32_t slot) { g_fault_snapshot[slot] = atomicExch(&g_fault_word, 0u); }

// ---------------------------------------------------------------------------
// conversion kernel (kvq_convert)
// ---------------------------------------------------------------------------
__global__ void convert_kernel(int32_t fmt, const float* in, int64_t n, uint8_t* out) {
    pdl_wait();
    pdl_trigger();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float v = in[i];
        switch (fmt) {
            case 0: out[i] = (uint8_t)e4m3x2(v, 0.0f); break;
            case 1: out[i] = (uint8_t)e5m2x2(v, 0.0f); break;
            case 2: {
                const float q[8] = {v, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                out[i] = (uint8_t)(e2m1x8(q) & 0xfu);
                break;
            }
            case 3: reinterpret_cast<uint16_t*>(out)[i] = (uint16_t)to_bf16_bits(v); break;
            case 4: out[i] = (uint8_t)e8m0_ceil(v); break;
            default: out[i] = (uint8_t)int8_rne_sat(v); break;
        }
    }
}

// ---------------------------------------------------------------------------
// self-test of the division shortcut (kvq_selftest)
// ---------------------------------------------------------------------------
__device__ unsigned long long g_selftest_count;

// grid.x: numerator bit patterns (65536); threads walk the scale patterns with
// biased exponent 27..227 (2^-100 <= s < 2^101), all 128 fractions each.
__global__ void selftest_div_kernel(int32_t which) {
    const uint32_t abits = blockIdx.x;
    if ((abits & 0x7f80u) == 0x7f80u) return;               // inf / NaN numerators
    const float a = __uint_as_float(abits << 16);
    unsigned long long bad = 0;
    for (uint32_t k = threadIdx.x; k < 201u * 128u; k += blockDim.x) {
        const uint32_t sbits = ((27u + k / 128u) << 7) | (k % 128u);
        const float s = __uint_as_float(sbits << 16);
        if (fabsf(a) > 512.0f * s) continue;
        const float r = __frcp_rn(s);
        const float ref = __fdiv_rn(a, s);
        float q1, q1b, t1, t1b;
        div_scale1_x2(a, -a, s, r, q1, q1b);        // the packed forms the kernels use
        div_scale1_neg_x2(a, -a, s, r, t1, t1b);
        if (__float_as_uint(q1b) != (__float_as_uint(q1) ^ 0x80000000u) ||
            __float_as_uint(t1) != (__float_as_uint(q1) ^ 0x80000000u) ||
            __float_as_uint(t1b) != (__float_as_uint(q1b) ^ 0x80000000u)) {
            atomicAdd(&g_selftest_count, 1ull);  // both halves and both forms must agree up to sign
        }
        bool diff;
        switch (which) {
            case 0: diff = __float_as_uint(q1) != __float_as_uint(ref); break;
            case 5: diff = fabsf(ref) >= 1.17549435e-38f && __float_as_uint(q1) != __float_as_uint(ref); break;
            case 1: diff = __float_as_uint(div_scale2(a, s, r)) != __float_as_uint(ref); break;
            case 2: {
                const uint32_t c = e4m3x2(ref, 0.0f);
                diff = e4m3x2(q1, 0.0f) != c || (e4m3x2(t1, 0.0f) ^ 0x80u) != c;
                break;
            }
            default: {
                const float v1[8] = {q1, t1, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                const float v2[8] = {ref, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                const uint32_t c1 = e2m1x8(v1), c2 = e2m1x8(v2) & 0xfu;
                diff = (c1 & 0xfu) != c2 || (((c1 >> 4) & 0xfu) ^ 0x8u) != c2;
            }
        }
        bad += diff ? 1ull : 0ull;
    }
    if (bad) atomicAdd(&g_selftest_count, bad);
}

// The fast int8 quantisation of the dequant kernel (int8x4_quant) against
// IEEE division on 2^28 random (o, scale, offset) triples per call: o of random
// sign and binade in [2^-70, 2^70], scale in [2^-70, 2^70], offset 0, a small
// integer, or a random value up to 2^17; half of the o values are placed within
// a few ulps of a rounding tie (o = (k + 1/2 - offset) * scale, k in
// [-140, 140]).  Counter-based hash (SplitMix64 finaliser) for the draws.
__device__ __forceinline__ uint64_t st_mix(uint64_t z) {
    z += 0x9e3779b97f4a7c15ull;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ float st_float(uint64_t h, int emin, int emax) {
    const int e = emin + (int)((h >> 40) % (uint64_t)(emax - emin + 1));
    const uint32_t m = (uint32_t)h & 0x7fffffu;
    return __uint_as_float(((uint32_t)(e + 127) << 23) | m);
}

__global__ void selftest_int8_kernel() {
    const uint64_t i0 = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) * 16u;
    unsigned long long bad = 0;
    for (uint64_t i = i0; i < i0 + 16u; i += 4u) {
        float o[4], sc[4], of[4], r[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint64_t h1 = st_mix(4 * (i + k)), h2 = st_mix(4 * (i + k) + 1), h3 = st_mix(4 * (i + k) + 2),
                           h4 = st_mix(4 * (i + k) + 3);
            sc[k] = st_float(h2, -70, 70);
            const uint32_t kind = (uint32_t)(h3 & 3u);
            of[k] = kind == 0 ? 0.0f : (kind == 1 ? (float)((int)((h3 >> 8) % 17u) - 8)
                                                  : st_float(h3 >> 2, -20, 17) * ((h3 >> 60) & 1u ? -1.0f : 1.0f));
            if (h4 & 1u) {
                const float tk = (float)((int)((h4 >> 8) % 281u) - 140);
                float v = __fmul_rn(__fadd_rn(__fadd_rn(tk, 0.5f), -of[k]), sc[k]);
                const int nudge = (int)((h4 >> 20) % 5u) - 2;
                v = __uint_as_float(__float_as_uint(v) + nudge);
                o[k] = v;
            } else {
                o[k] = st_float(h1, -70, 70) * ((h1 >> 63) ? -1.0f : 1.0f);
            }
            r[k] = int8_quant_rcp(sc[k], of[k]);
        }
        const uint32_t fast = int8x4_quant(o, sc, of, r);
        uint32_t ref = 0u;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            ref |= ((uint32_t)int8_rne_sat(__fadd_rn(__fdiv_rn(o[k], sc[k]), of[k])) & 0xffu) << (8 * k);
        bad += fast != ref ? 1ull : 0ull;
    }
    if (bad) atomicAdd(&g_selftest_count, bad);
}

// The bounded wait of the pipelined kernels running out: one warp waits on
// an mbarrier that nothing arrives on, with a short limit; the wait must
// return false (counted) and set FAULT_TIMEOUT in the fault word.  The CTA
// then exits normally -- no GPU fault, hang or trap is involved.
__global__ void selftest_timeout_kernel() {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_init_fence();
    }
    __syncthreads();
    const bool done = __all_sync(FULL_MASK, mbar_wait(&bar, 0u, 4096u));
    if (threadIdx.x == 0 && !done) atomicAdd(&g_selftest_count, 1ull);
}

// The indexer's fp8 mode: codes from the two-step quotient (where
// ix_fp8_fast admits the row maximum) against codes from IEEE division, for
// 2^28 random (x, amax) pairs per call: amax a random finite bf16 (as bits)
// of binade 2^-70 .. 2^127 or f16 (alternating calls' halves), x a random
// value of the same type with |x| <= amax (every binade down to the
// subnormals, zeros of both signs included), E4M3 and E5M2 codes; counts the
// pairs whose codes differ.
__global__ void selftest_fp8_row_kernel() {
    const uint64_t i0 = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) * 16u;
    unsigned long long bad = 0;
    for (uint64_t i = i0; i < i0 + 16u; ++i) {
        const uint64_t h1 = st_mix(2 * i), h2 = st_mix(2 * i + 1);
        const bool f16 = (i >> 20) & 1u;
        float amax, x;
        if (f16) {
            const uint32_t ab = 1u + (uint32_t)(h1 % 0x7bffu);                      // (0, 65504]
            amax = __half2float(__ushort_as_half((unsigned short)ab));
            const uint32_t xb = (uint32_t)((h2 >> 8) % (ab + 1u)) | ((uint32_t)(h2 & 1u) << 15);
            x = __half2float(__ushort_as_half((unsigned short)xb));
        } else {
            const uint32_t ab = 0x0880u + (uint32_t)(h1 % (0x7f80u - 0x0880u));    // [~2^-111, max bf16]
            amax = __uint_as_float(ab << 16);
            const uint32_t xb = (uint32_t)((h2 >> 8) % (ab + 1u)) | ((uint32_t)(h2 & 1u) << 15);
            x = __uint_as_float(xb << 16);
        }
        if (!kvq::ix_fp8_fast(amax)) continue;
#pragma unroll
        for (int e5 = 0; e5 < 2; ++e5) {
            const float fmax = e5 ? 57344.0f : 448.0f;
            const float s = div_by_fmax(amax, fmax);
            const float q2 = div_scale2(x, s, __frcp_rn(s));
            const float qi = __fdiv_rn(x, s);
            const uint32_t c2 = e5 ? fp8x2<true>(q2, 0.0f) : fp8x2<false>(q2, 0.0f);
            const uint32_t ci = e5 ? fp8x2<true>(qi, 0.0f) : fp8x2<false>(qi, 0.0f);
            bad += c2 != ci ? 1ull : 0ull;
        }
    }
    if (bad) atomicAdd(&g_selftest_count, bad);
}

// The one-step quotient of the rmsnorm kernels (div1_x2_nz with r =
// RN(1/rms), numerators never zero) against IEEE division, 2^28 random pairs
// per call: rms a random
// binary32 of binade 2^-60 .. 2^49; x a random bf16 of either sign with |x| of
// binade max(e(rms) - 124, -103) .. e(rms) + 12; for half of the pairs rms is
// then replaced by RN(x / t) nudged by up to two ulps, t halfway between
// x / rms and its next binary32 value, so that x / rms lies within a few ulps
// of a rounding tie.  Pairs outside the kernel's guard (rms in [2^-60, 2^50],
// |x| >= max(RN(rms 2^-125), 2^-103)) are skipped; counts the pairs whose
// quotient (of x and of -x) differs from the IEEE quotient in any bit.
__global__ void selftest_rms_quot_kernel() {
    const uint64_t i0 = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) * 16u;
    unsigned long long bad = 0;
    for (uint64_t i = i0; i < i0 + 16u; ++i) {
        const uint64_t h1 = st_mix(3 * i), h2 = st_mix(3 * i + 1), h3 = st_mix(3 * i + 2);
        float rms = st_float(h1, -60, 49);
        const int er = (int)((__float_as_uint(rms) >> 23) & 0xffu) - 127;
        const int lo = er - 124 > -103 ? er - 124 : -103, hi = er + 12;
        const int ex = lo + (int)((h2 >> 8) % (uint64_t)(hi - lo + 1));
        const uint32_t xb = ((uint32_t)(ex + 127) << 23) | ((uint32_t)(h2 & 0x7fu) << 16) |
                            ((uint32_t)((h2 >> 7) & 1u) << 31);
        const float x = __uint_as_float(xb);
        if (h3 & 1u) {
            const float q = __fdiv_rn(x, rms);
            const double qa = fabs((double)q);
            const double t = 0.5 * (qa + (double)__uint_as_float(__float_as_uint((float)qa) + 1u));
            float r2 = (float)(fabs((double)x) / t);
            r2 = __uint_as_float(__float_as_uint(r2) + (uint32_t)((int)((h3 >> 8) % 5u) - 2));
            rms = r2;
        }
        if (!(rms >= 8.673617379884035e-19f && rms <= 1.125899906842624e15f)) continue;
        const float thr = fmaxf(__fmul_rn(rms, 2.350988701644575e-38f), 9.860761315262648e-32f);
        if (fabsf(x) < thr) continue;
        float q0, q1;
        div1_x2_nz(x, -x, rms, __frcp_rn(rms), q0, q1);
        const float ref = __fdiv_rn(x, rms);
        bad += (__float_as_uint(q0) != __float_as_uint(ref) || __float_as_uint(q1) != __float_as_uint(-ref)) ? 1ull
                                                                                                              : 0ull;
    }
    if (bad) atomicAdd(&g_selftest_count, bad);
}

// The one-step quotient (div1_x2_nz) of every bf16 and every f16 numerator
// mantissa, of both signs, by every binary32 divisor mantissa (one thread per
// divisor, 2^23 threads), numerator and divisor in [1, 2): counts the pairs
// whose quotient differs in any bit from IEEE division.  Scaling numerator and
// divisor by powers of two scales every intermediate exactly while they stay
// normal, so this covers every pair whose reciprocal, quotient and residual
// are normal.
__global__ void selftest_quot_mant_kernel() {
    const uint32_t j = blockIdx.x * blockDim.x + threadIdx.x;       // 0 .. 2^23 - 1
    const float b = __uint_as_float(0x3f800000u | (j & 0x7fffffu));
    const float r = __frcp_rn(b);
    unsigned long long bad = 0;
    for (uint32_t i = 0; i < 128u + 1024u; ++i) {
        const uint32_t m = i < 128u ? i << 16 : (i - 128u) << 13;   // bf16: 7 fraction bits, f16: 10
        const float x = __uint_as_float(0x3f800000u | m);
        float q0, q1;
        div1_x2_nz(x, -x, b, r, q0, q1);
        const float ref = __fdiv_rn(x, b);
        bad += (__float_as_uint(q0) != __float_as_uint(ref) || __float_as_uint(q1) != __float_as_uint(-ref)) ? 1ull
                                                                                                              : 0ull;
    }
    if (bad) atomicAdd(&g_selftest_count, bad);
}

// every positive finite bf16 amax (bits < 0x7f80) and every positive finite
// f16 amax (bits < 0x7c00) over the three format maxima
__global__ void selftest_fmax_kernel() {
    const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;       // 0 .. 65535
    const uint32_t bits = i & 0x7fffu;
    const bool f16 = i >= 0x8000u;
    if (bits >= (f16 ? 0x7c00u : 0x7f80u)) return;
    const float a = f16 ? __half2float(__ushort_as_half((unsigned short)bits)) : __uint_as_float(bits << 16);
    unsigned long long bad = 0;
    const float cs[3] = {448.0f, 57344.0f, 6.0f};
#pragma unroll
    for (int i = 0; i < 3; ++i)
        bad += __float_as_uint(div_by_fmax(a, cs[i])) != __float_as_uint(__fdiv_rn(a, cs[i])) ? 1ull : 0ull;
    if (bad) atomicAdd(&g_selftest_count, bad);
}

// The pipelined dequant kernel instantiated for the ring shape (a.stages,
// a.tps) that the host picked, and for D = 128 or any other head size.
template <int XK, bool F16, int S, int TPS>
cudaError_t launch_drq_tma(const DrqArgs& a, int64_t tiles, size_t smem, cudaStream_t s) {
    auto k = a.D == 128 ? dequant_rope_quant_tma_kernel<XK, F16, S, TPS, 128>
                        : dequant_rope_quant_tma_kernel<XK, F16, S, TPS, 0>;
    return launch(k, (unsigned)persistent_grid(k, DT_THREADS, tiles, smem), DT_THREADS, smem, s, a);
}

template <int XK, bool F16, int S>
cudaError_t launch_drq_tps(const DrqArgs& a, int64_t tiles, size_t smem, cudaStream_t s) {
    if (a.tps == 2) return launch_drq_tma<XK, F16, S, 2>(a, tiles, smem, s);
    if (a.tps == 4) return launch_drq_tma<XK, F16, S, 4>(a, tiles, smem, s);
    return launch_drq_tma<XK, F16, S, 8>(a, tiles, smem, s);
}

template <int XK, bool F16>
cudaError_t launch_drq_ring(const DrqArgs& a, int64_t tiles, size_t smem, cudaStream_t s) {
    if (a.stages == 2) return launch_drq_tps<XK, F16, 2>(a, tiles, smem, s);
    if (a.stages == 3) return launch_drq_tps<XK, F16, 3>(a, tiles, smem, s);
    return launch_drq_tps<XK, F16, 4>(a, tiles, smem, s);
}

}  // namespace

extern "C" {

kvq_status kvq_selftest(int32_t which, uint64_t* result, kvq_stream stream) {
    if (!result) return KVQ_ERR_NULL;
    if (which < 0 || which > 10) return KVQ_ERR_ATTR;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const unsigned long long zero = 0ull;
    unsigned long long h = 0ull;
    if (cudaMemcpyToSymbolAsync(g_selftest_count, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return KVQ_ERR_CUDA;
    if (which == 4) selftest_fmax_kernel<<<256, 256, 0, s>>>();
    else if (which == 6) selftest_int8_kernel<<<65536, 256, 0, s>>>();
    else if (which == 7) selftest_timeout_kernel<<<1, 32, 0, s>>>();
    else if (which == 8) selftest_fp8_row_kernel<<<65536, 256, 0, s>>>();
    else if (which == 9) selftest_rms_quot_kernel<<<65536, 256, 0, s>>>();
    else if (which == 10) selftest_quot_mant_kernel<<<(1u << 23) / 256u, 256, 0, s>>>();
    else selftest_div_kernel<<<65536, 256, 0, s>>>(which);
    if (cudaGetLastError() != cudaSuccess) return KVQ_ERR_CUDA;
    if (cudaMemcpyFromSymbolAsync(&h, g_selftest_count, sizeof(h), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return KVQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return KVQ_ERR_CUDA;
    *result = h;
    return KVQ_OK;
}

int32_t kvq_version(void) { return 100; }

const char* kvq_status_string(kvq_status s) {
    switch (s) {
        case KVQ_OK: return "ok";
        case KVQ_ERR_NULL: return "a required tensor or data pointer is NULL";
        case KVQ_ERR_NDIM: return "wrong number of dimensions";
        case KVQ_ERR_SHAPE: return "inconsistent tensor sizes";
        case KVQ_ERR_DTYPE: return "dtype not allowed";
        case KVQ_ERR_ATTR: return "bad attribute value";
        case KVQ_ERR_LAYOUT: return "non-contiguous where contiguity is required";
        case KVQ_ERR_CAPACITY: return "cache row too small for the packed row";
        case KVQ_ERR_CUDA: return "CUDA runtime error";
        case KVQ_ERR_UNSUPPORTED: return "valid but not implemented by this library";
        default: return "unknown status";
    }
}

int64_t kvq_kv_cache_col(int64_t d, int32_t quant_mode, int32_t quant_group_size) {
    if (d <= 64 || d % 64 != 0 || d > 8192) return -1;
    const int64_t n = d - 64;
    int64_t concat;
    if (quant_mode == 0 || quant_mode == 1) {
        concat = n + 128 + ((n + 63) / 64) * (quant_mode == 0 ? 2 : 1);
    } else if (quant_mode == 2) {
        if (quant_group_size != 16 && quant_group_size != 32 && quant_group_size != 64) return -1;
        if (n % quant_group_size != 0) return -1;
        concat = 64 + n / 2 + (n / quant_group_size) * 2;
    } else {
        return -1;
    }
    return quant_mode == 1 ? concat : (concat + 31) / 32 * 32;
}

int64_t kvq_indexer_scale_col(int64_t d, int32_t quant_mode) {
    if (d < 1) return -1;
    if (quant_mode == 0 || quant_mode == 3) return (d + 31) / 32;
    if (quant_mode == 1 || quant_mode == 2) return 1;
    return -1;
}

// ---------------------------------------------------------------------------
kvq_status kvq_kv_compress_epilog(const kvq_tensor* x, const kvq_tensor* slot_mapping, kvq_tensor* cache,
                                  int32_t quant_mode, int32_t quant_group_size, float x_scale,
                                  kvq_stream stream) {
    Trace trace("kvq_kv_compress_epilog");
    if (!x || !slot_mapping || !cache) return KVQ_ERR_NULL;
    if (!valid_desc(x) || !valid_desc(slot_mapping) || !valid_desc(cache)) return KVQ_ERR_DTYPE;
    if (x->dtype != KVQ_BF16 && x->dtype != KVQ_F16) return KVQ_ERR_DTYPE;
    if (x->ndim < 1) return KVQ_ERR_NDIM;
    int64_t T, rs;
    if (!flatten_rows(x, &T, &rs)) return KVQ_ERR_LAYOUT;
    const int64_t d = x->shape[x->ndim - 1];
    if (d <= 64 || d % 64 != 0 || d > 8192) return KVQ_ERR_SHAPE;
    if (quant_mode < 0 || quant_mode > 2) return KVQ_ERR_ATTR;
    if (quant_mode == 2 && x->dtype != KVQ_BF16) return KVQ_ERR_DTYPE;     // mode 2 needs bf16 x
    const bool xf16 = x->dtype == KVQ_F16;
    const int32_t G = quant_mode == 2 ? quant_group_size : 64;
    if (quant_mode == 2 && ((G != 16 && G != 32 && G != 64) || (d - 64) % G != 0)) return KVQ_ERR_ATTR;
    if (!is_index_dtype(slot_mapping->dtype)) return KVQ_ERR_DTYPE;
    if (numel(slot_mapping) != T) return KVQ_ERR_SHAPE;
    if (!contiguous(slot_mapping)) return KVQ_ERR_LAYOUT;
    if (cache->dtype != KVQ_U8 && cache->dtype != KVQ_I8) return KVQ_ERR_DTYPE;
    if (cache->ndim != 4) return KVQ_ERR_NDIM;
    if (cache->shape[2] != 1) return KVQ_ERR_SHAPE;
    PagedRows rows;
    int64_t head_dim;
    kvq_status st = paged_from(cache, 1, &rows, &head_dim);
    if (st != KVQ_OK) return st;
    const int64_t col = kvq_kv_cache_col(d, quant_mode, G);
    if (head_dim < col) return KVQ_ERR_CAPACITY;
    if (T == 0) return KVQ_OK;
    if (!x->data || !slot_mapping->data || (!cache->data && rows.num_slots > 0)) return KVQ_ERR_NULL;

    CompressArgs a;
    a.x = static_cast<const uint16_t*>(x->data);
    a.x_row_stride = rs;
    a.T = T;
    a.slots = slot_mapping->data;
    a.slots_i64 = slot_mapping->dtype == KVQ_I64;
    a.cache = rows;
    a.nseg = (int32_t)(d / 64);
    a.n = (int32_t)(d - 64);
    a.col = (int32_t)col;
    a.concat = quant_mode == 2 ? (int32_t)(64 + (d - 64) / 2 + ((d - 64) / G) * 2)
                               : (int32_t)((d - 64) + 128 + ((d - 64) / 64) * (quant_mode == 0 ? 2 : 1));
    a.x_scale = x_scale;
    a.x_vec = (reinterpret_cast<uintptr_t>(x->data) % 16 == 0) && ((rs * 2) % 16 == 0);

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // pipelined kernel when x rows are 16-byte aligned and a ring of at least
    // two 32-row stages fits in shared memory (d <= 1728); else the direct one
    const size_t smem_limit = 227 * 1024;
    const bool rows_aligned = (reinterpret_cast<uintptr_t>(cache->data) % 16 == 0) && rows.row_bytes % 16 == 0 &&
                              rows.block_stride % 16 == 0;
    // packed rows leave by bulk copy when the rows are aligned, kvCacheCol is a
    // multiple of 16 and each consumer warp owns one segment (d <= 1024); two
    // input stages and one output buffer then keep two CTAs on an SM
    const bool bulk_out = rows_aligned && col % 16 == 0 && d / 64 <= CT_MAX_CONSUMER_WARPS;
    auto ct_smem = [&](int stages) {
        return ct_header_bytes(stages) + (size_t)stages * CT_ROWS * ct_pitch((int)(d / 64)) +
               (bulk_out ? (size_t)CT_ROWS * ct_out_pitch((int)col) : 0);
    };
    const int want = bulk_out ? 2 : 3;
    const int ct_stages = ct_smem(want) <= smem_limit ? want : (ct_smem(2) <= smem_limit ? 2 : 0);
    // decode-sized batches (fewer rows than one 32-row tile per SM) take the
    // direct kernel: no pipeline to fill, one load-compute-store round trip
    const bool small = T < 32 * (int64_t)sm_count();
    if (a.x_vec && ct_stages > 0 && !small) {
        // pipelined kernel: rows arrive in shared memory by bulk copy
        a.ncw = a.nseg < CT_MAX_CONSUMER_WARPS ? a.nseg : CT_MAX_CONSUMER_WARPS;
        a.stages = ct_stages;
        a.rows_aligned = rows_aligned;
        a.bulk_out = bulk_out;
        const size_t smem = ct_smem(ct_stages);
        const int64_t tiles = (T + CT_ROWS - 1) / CT_ROWS;
        const int threads = (a.ncw + 1) * 32;
        cudaError_t err = cudaSuccess;
#define KVQ_LAUNCH_CT(M, GG, F)                                                                \
    do {                                                                                       \
        auto k = ct_stages == 2 ? compress_tma_kernel<M, GG, 2, F> : compress_tma_kernel<M, GG, 3, F>; \
        err = launch(k, (unsigned)persistent_grid(k, threads, tiles, smem), threads, smem, s, a); \
    } while (0)
        if (quant_mode == 0) {
            if (xf16) KVQ_LAUNCH_CT(0, 64, true);
            else KVQ_LAUNCH_CT(0, 64, false);
        } else if (quant_mode == 1) {
            if (xf16) KVQ_LAUNCH_CT(1, 64, true);
            else KVQ_LAUNCH_CT(1, 64, false);
        } else if (G == 16) KVQ_LAUNCH_CT(2, 16, false);
        else if (G == 32) KVQ_LAUNCH_CT(2, 32, false);
        else KVQ_LAUNCH_CT(2, 64, false);
#undef KVQ_LAUNCH_CT
        return launched(err);
    }
    {
        const int64_t r = (4 * CE_UNROLL) / a.nseg;       // rows whose segments fill one round
        a.ce_rows = (int32_t)(r < 1 ? 1 : (r > CE_TILE ? CE_TILE : r));
    }
    const int64_t tiles = (T + a.ce_rows - 1) / a.ce_rows;
    const int64_t need = (tiles + (CE_THREADS / 32) - 1) / (CE_THREADS / 32);
    cudaError_t err = cudaSuccess;
#define KVQ_LAUNCH_CE(M, GG, F)                                                                \
    do {                                                                                       \
        auto k = compress_epilog_kernel<M, GG, F>;                                             \
        err = launch(k, (unsigned)persistent_grid(k, CE_THREADS, need), CE_THREADS, 0, s, a);    \
    } while (0)
    if (quant_mode == 0) {
        if (xf16) KVQ_LAUNCH_CE(0, 64, true);
        else KVQ_LAUNCH_CE(0, 64, false);
    } else if (quant_mode == 1) {
        if (xf16) KVQ_LAUNCH_CE(1, 64, true);
        else KVQ_LAUNCH_CE(1, 64, false);
    } else if (G == 16) KVQ_LAUNCH_CE(2, 16, false);
    else if (G == 32) KVQ_LAUNCH_CE(2, 32, false);
    else KVQ_LAUNCH_CE(2, 64, false);
#undef KVQ_LAUNCH_CE
    return launched(err);
}

// ---------------------------------------------------------------------------
kvq_status kvq_kv_decompress(const kvq_tensor* cache, const kvq_tensor* slot_mapping, kvq_tensor* y,
                             int32_t quant_mode, int32_t quant_group_size, float x_scale, kvq_stream stream) {
    Trace trace("kvq_kv_decompress");
    if (!cache || !slot_mapping || !y) return KVQ_ERR_NULL;
    if (!valid_desc(cache) || !valid_desc(slot_mapping) || !valid_desc(y)) return KVQ_ERR_DTYPE;
    if (y->dtype != KVQ_BF16 && y->dtype != KVQ_F16) return KVQ_ERR_DTYPE;
    if (quant_mode == 2 && y->dtype != KVQ_BF16) return KVQ_ERR_DTYPE;     // mode 2 rows come from bf16 x
    const bool yf16 = y->dtype == KVQ_F16;
    if (y->ndim < 1) return KVQ_ERR_NDIM;
    int64_t T, ys;
    if (!flatten_rows(y, &T, &ys)) return KVQ_ERR_LAYOUT;
    const int64_t d = y->shape[y->ndim - 1];
    if (d <= 64 || d % 64 != 0 || d > 8192) return KVQ_ERR_SHAPE;
    if (quant_mode < 0 || quant_mode > 2) return KVQ_ERR_ATTR;
    const int32_t G = quant_mode == 2 ? quant_group_size : 64;
    if (quant_mode == 2 && ((G != 16 && G != 32 && G != 64) || (d - 64) % G != 0)) return KVQ_ERR_ATTR;
    if (!is_index_dtype(slot_mapping->dtype)) return KVQ_ERR_DTYPE;
    if (numel(slot_mapping) != T) return KVQ_ERR_SHAPE;
    if (!contiguous(slot_mapping)) return KVQ_ERR_LAYOUT;
    if (cache->dtype != KVQ_U8 && cache->dtype != KVQ_I8) return KVQ_ERR_DTYPE;
    if (cache->ndim != 4) return KVQ_ERR_NDIM;
    if (cache->shape[2] != 1) return KVQ_ERR_SHAPE;
    PagedRows rows;
    int64_t head_dim;
    kvq_status st = paged_from(cache, 1, &rows, &head_dim);
    if (st != KVQ_OK) return st;
    if (head_dim < kvq_kv_cache_col(d, quant_mode, G)) return KVQ_ERR_CAPACITY;
    if (T == 0) return KVQ_OK;
    if (!y->data || !slot_mapping->data || (!cache->data && rows.num_slots > 0)) return KVQ_ERR_NULL;

    DecompressArgs a;
    a.cache = rows;
    a.slots = slot_mapping->data;
    a.slots_i64 = slot_mapping->dtype == KVQ_I64;
    a.T = T;
    a.y = static_cast<uint16_t*>(y->data);
    a.y_row_stride = ys;
    a.nslice = (int32_t)(d / 32);
    a.n = (int32_t)(d - 64);
    a.x_scale = x_scale;
    a.rows_vec16 = (reinterpret_cast<uintptr_t>(cache->data) % 16 == 0) && rows.row_bytes % 16 == 0 &&
                   rows.block_stride % 16 == 0;
    a.y_vec32 = (reinterpret_cast<uintptr_t>(y->data) % 32 == 0) && (ys * 2) % 32 == 0;
    const int64_t nn = a.nslice - 2;
    const bool dbl = quant_mode == 2 && G >= 32 && nn % 4 == 0;            // see kv_decompress_kernel
    const int64_t nchunks = quant_mode == 2 ? ((T + 15) / 16) * ((dbl ? nn / 4 : nn / 2) + 1)
                                            : (T * a.nslice + 31) / 32;
    const int64_t need = (nchunks + (DC_THREADS / 32) - 1) / (DC_THREADS / 32);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t err = cudaSuccess;
#define KVQ_LAUNCH_DC(M, GG, F)                                                                \
    do {                                                                                       \
        auto k = a.nslice == 18 ? kv_decompress_kernel<M, GG, 18, F> : kv_decompress_kernel<M, GG, 0, F>; \
        err = launch(k, (unsigned)persistent_grid(k, DC_THREADS, need), DC_THREADS, 0, s, a);    \
    } while (0)
    if (quant_mode == 0) {
        if (yf16) KVQ_LAUNCH_DC(0, 64, true);
        else KVQ_LAUNCH_DC(0, 64, false);
    } else if (quant_mode == 1) {
        if (yf16) KVQ_LAUNCH_DC(1, 64, true);
        else KVQ_LAUNCH_DC(1, 64, false);
    } else if (G == 16) {
        KVQ_LAUNCH_DC(2, 16, false);
    } else {
        auto run2 = [&](auto kernel) {
            return launch(kernel, (unsigned)persistent_grid(kernel, DC_THREADS, need), DC_THREADS, 0, s, a);
        };
        if (G == 32) err = dbl ? (a.nslice == 18 ? run2(kv_decompress_kernel<2, 32, 18, false, true>)
                                                 : run2(kv_decompress_kernel<2, 32, 0, false, true>))
                               : (a.nslice == 18 ? run2(kv_decompress_kernel<2, 32, 18, false, false>)
                                                 : run2(kv_decompress_kernel<2, 32, 0, false, false>));
        else err = dbl ? (a.nslice == 18 ? run2(kv_decompress_kernel<2, 64, 18, false, true>)
                                         : run2(kv_decompress_kernel<2, 64, 0, false, true>))
                       : (a.nslice == 18 ? run2(kv_decompress_kernel<2, 64, 18, false, false>)
                                         : run2(kv_decompress_kernel<2, 64, 0, false, false>));
    }
#undef KVQ_LAUNCH_DC
    return launched(err);
}

kvq_status kvq_indexer_quant_cache(const kvq_tensor* x, kvq_tensor* cache, kvq_tensor* cache_scale,
                                   const kvq_tensor* slot_mapping, int32_t quant_mode, kvq_stream stream) {
    Trace trace("kvq_indexer_quant_cache");
    if (!x || !cache || !cache_scale || !slot_mapping) return KVQ_ERR_NULL;
    if (!valid_desc(x) || !valid_desc(cache) || !valid_desc(cache_scale) || !valid_desc(slot_mapping))
        return KVQ_ERR_DTYPE;
    if (x->dtype != KVQ_BF16 && x->dtype != KVQ_F16) return KVQ_ERR_DTYPE;
    if (x->ndim < 1) return KVQ_ERR_NDIM;
    int64_t T, rs;
    if (!flatten_rows(x, &T, &rs)) return KVQ_ERR_LAYOUT;
    const int64_t d = x->shape[x->ndim - 1];
    if (d < 1 || d > (1 << 24)) return KVQ_ERR_SHAPE;    // the kernel indexes a row with 32-bit integers
    if (quant_mode == 2) return KVQ_ERR_UNSUPPORTED;
    if (quant_mode != 0 && quant_mode != 1 && quant_mode != 3) return KVQ_ERR_ATTR;
    if (quant_mode == 3) {
        if (cache->dtype != KVQ_U8 && cache->dtype != KVQ_I8) return KVQ_ERR_DTYPE;
    } else if (cache->dtype != KVQ_F8E4M3 && cache->dtype != KVQ_F8E5M2) {
        return KVQ_ERR_DTYPE;
    }
    if (quant_mode == 1) {
        if (cache_scale->dtype != KVQ_F32) return KVQ_ERR_DTYPE;
    } else if (cache_scale->dtype != KVQ_E8M0 && cache_scale->dtype != KVQ_U8) {
        return KVQ_ERR_DTYPE;
    }
    if (!is_index_dtype(slot_mapping->dtype)) return KVQ_ERR_DTYPE;
    if (numel(slot_mapping) != T) return KVQ_ERR_SHAPE;
    if (!contiguous(slot_mapping)) return KVQ_ERR_LAYOUT;
    if (cache->ndim != 4 || cache_scale->ndim != 4) return KVQ_ERR_NDIM;
    if (cache->shape[2] != 1 || cache_scale->shape[2] != 1) return KVQ_ERR_SHAPE;
    PagedRows crow, srow;
    int64_t chd, shd;
    kvq_status st = paged_from(cache, 1, &crow, &chd);
    if (st != KVQ_OK) return st;
    st = paged_from(cache_scale, 1, &srow, &shd);
    if (st != KVQ_OK) return st;
    if (cache->shape[0] != cache_scale->shape[0] || cache->shape[1] != cache_scale->shape[1]) return KVQ_ERR_SHAPE;
    const int64_t need_codes = quant_mode == 3 ? (d + 1) / 2 : d;
    if (chd < need_codes || shd < kvq_indexer_scale_col(d, quant_mode)) return KVQ_ERR_CAPACITY;
    if (T == 0) return KVQ_OK;
    if (!x->data || !slot_mapping->data || !cache->data || !cache_scale->data) return KVQ_ERR_NULL;

    IndexerArgs a;
    a.x = static_cast<const uint16_t*>(x->data);
    a.x_row_stride = rs;
    a.T = T;
    a.d = (int32_t)d;
    a.ngroups = (int32_t)((d + 31) / 32);
    a.team_shift = 0;
    while ((1 << a.team_shift) < a.ngroups && a.team_shift < 5) ++a.team_shift;
    const uintptr_t xa = reinterpret_cast<uintptr_t>(x->data);
    a.x_vec = (xa % 32 == 0 && (rs * 2) % 32 == 0) ? 2 : ((xa % 16 == 0 && (rs * 2) % 16 == 0) ? 1 : 0);
    a.slots = slot_mapping->data;
    a.slots_i64 = slot_mapping->dtype == KVQ_I64;
    a.cache = crow;
    a.scale = srow;
    a.code_vec32 = (reinterpret_cast<uintptr_t>(cache->data) % 32 == 0) && crow.row_bytes % 32 == 0 &&
                   crow.block_stride % 32 == 0;
    const bool f16 = x->dtype == KVQ_F16, e5m2 = cache->dtype == KVQ_F8E5M2;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t passes = (T + (32 >> a.team_shift) - 1) / (32 >> a.team_shift);
    const int64_t need = (passes + (IX_THREADS / 32) - 1) / (IX_THREADS / 32);
    cudaError_t err = cudaSuccess;
#define KVQ_LAUNCH_IX(M, F, E)                                                                 \
    do {                                                                                       \
        auto k = indexer_quant_kernel<M, F, E>;                                                \
        err = launch(k, (unsigned)persistent_grid(k, IX_THREADS, need), IX_THREADS, 0, s, a);    \
    } while (0)
#define KVQ_LAUNCH_IX_FE(M)                                                                    \
    do {                                                                                       \
        if (f16) {                                                                             \
            if (e5m2) KVQ_LAUNCH_IX(M, true, true);                                            \
            else KVQ_LAUNCH_IX(M, true, false);                                                \
        } else {                                                                               \
            if (e5m2) KVQ_LAUNCH_IX(M, false, true);                                           \
            else KVQ_LAUNCH_IX(M, false, false);                                               \
        }                                                                                      \
    } while (0)
    if (quant_mode == 0) KVQ_LAUNCH_IX_FE(0);
    else if (quant_mode == 1) KVQ_LAUNCH_IX_FE(1);
    else if (f16) KVQ_LAUNCH_IX(3, true, false);
    else KVQ_LAUNCH_IX(3, false, false);
#undef KVQ_LAUNCH_IX_FE
#undef KVQ_LAUNCH_IX
    return launched(err);
}

// ---------------------------------------------------------------------------
namespace {

int32_t cache_dt(int32_t dt) {
    switch (dt) {
        case KVQ_BF16: return CDT_BF16;
        case KVQ_F16: return CDT_F16;
        case KVQ_F8E4M3: return CDT_E4M3;
        case KVQ_F8E5M2: return CDT_E5M2;
        case KVQ_I8: return CDT_I8;
        default: return -1;
    }
}

// scale / offset of a quantised cache: f32, 1 or Dc elements, contiguous
kvq_status cache_param(const kvq_tensor* p, int64_t dc, const float** out, int32_t* n) {
    *out = nullptr;
    *n = 0;
    if (!p) return KVQ_OK;
    if (!valid_desc(p) || p->dtype != KVQ_F32) return KVQ_ERR_DTYPE;
    const int64_t k = numel(p);
    if (k != 1 && k != dc) return KVQ_ERR_SHAPE;
    if (!contiguous(p)) return KVQ_ERR_LAYOUT;
    *out = static_cast<const float*>(p->data);
    *n = (int32_t)k;
    return KVQ_OK;
}

kvq_status setup_cache_out(const kvq_tensor* c, const kvq_tensor* scale, const kvq_tensor* offset,
                           CacheOut* out, int64_t* head_dim) {
    if (!valid_desc(c)) return KVQ_ERR_DTYPE;
    out->dt = cache_dt(c->dtype);
    if (out->dt < 0) return KVQ_ERR_DTYPE;
    kvq_status st = paged_from(c, 1, &out->rows, head_dim);
    if (st != KVQ_OK) return st;
    const bool quant = out->dt == CDT_E4M3 || out->dt == CDT_E5M2 || out->dt == CDT_I8;
    if (quant && !scale) return KVQ_ERR_NULL;
    if (offset && out->dt != CDT_I8) return KVQ_ERR_ATTR;
    st = cache_param(quant ? scale : nullptr, *head_dim, &out->scale, &out->scale_n);
    if (st != KVQ_OK) return st;
    return cache_param(offset, *head_dim, &out->offset, &out->offset_n);
}

}  // namespace

kvq_status kvq_kv_rmsnorm_rope_cache(const kvq_tensor* kv, const kvq_tensor* gamma, const kvq_tensor* cos,
                                     const kvq_tensor* sin, const kvq_tensor* index, kvq_tensor* k_cache,
                                     kvq_tensor* ckv_cache, const kvq_tensor* k_scale,
                                     const kvq_tensor* ckv_scale, const kvq_tensor* k_offset,
                                     const kvq_tensor* ckv_offset, float epsilon, int32_t cache_mode,
                                     kvq_stream stream) {
    Trace trace("kvq_kv_rmsnorm_rope_cache");
    if (!kv || !gamma || !cos || !sin || !index || !k_cache || !ckv_cache) return KVQ_ERR_NULL;
    if (!valid_desc(kv) || !valid_desc(gamma) || !valid_desc(cos) || !valid_desc(sin) || !valid_desc(index))
        return KVQ_ERR_DTYPE;
    if (cache_mode == 4 || cache_mode == 5) return KVQ_ERR_UNSUPPORTED;   // PA_NZ, PA_BLK_NZ
    if (cache_mode < 0 || cache_mode > 3) return KVQ_ERR_ATTR;
    if (kv->dtype != KVQ_BF16 && kv->dtype != KVQ_F16) return KVQ_ERR_DTYPE;
    if (gamma->dtype != kv->dtype || cos->dtype != kv->dtype || sin->dtype != kv->dtype) return KVQ_ERR_DTYPE;
    if (kv->ndim != 4) return KVQ_ERR_NDIM;
    if (kv->shape[1] != 1) return KVQ_ERR_SHAPE;
    if (!contiguous(kv) || !contiguous(gamma) || !contiguous(cos) || !contiguous(sin) || !contiguous(index))
        return KVQ_ERR_LAYOUT;
    const int64_t B = kv->shape[0], S = kv->shape[2], D = kv->shape[3];
    CacheOut kc, cc;
    int64_t Dk, Dv;
    kvq_status st = setup_cache_out(k_cache, k_scale, k_offset, &kc, &Dk);
    if (st != KVQ_OK) return st;
    st = setup_cache_out(ckv_cache, ckv_scale, ckv_offset, &cc, &Dv);
    if (st != KVQ_OK) return st;
    if (Dk + Dv != D || Dk % 2 != 0 || Dk < 2 || Dv < 1) return KVQ_ERR_SHAPE;
    if (D > (1 << 24)) return KVQ_ERR_SHAPE;              // the kernel indexes a row with 32-bit integers
    const bool kq = kc.dt >= CDT_E4M3, cq = cc.dt >= CDT_E4M3;
    if (kq && cq && kc.dt != cc.dt) return KVQ_ERR_DTYPE;     // scenario 3 needs one dtype
    if (k_cache->shape[0] != ckv_cache->shape[0] || kc.rows.block_size != cc.rows.block_size) return KVQ_ERR_SHAPE;
    const int64_t bs = kc.rows.block_size;
    if (cache_mode != 0) {
        // PA block size rule: % 32 for 1-byte caches, % 16 for 2-byte ones
        const bool one_byte = kq || cq, two_byte = !kq || !cq;
        if ((one_byte && bs % 32 != 0) || (two_byte && bs % 16 != 0)) return KVQ_ERR_SHAPE;
    }
    if (numel(gamma) != Dv || numel(cos) != B * S * Dk || numel(sin) != B * S * Dk) return KVQ_ERR_SHAPE;
    if (!is_index_dtype(index->dtype)) return KVQ_ERR_DTYPE;
    const int64_t nidx = cache_mode == 3 ? B * ((S + bs - 1) / (bs > 0 ? bs : 1)) : B * S;
    if (numel(index) != nidx) return KVQ_ERR_SHAPE;
    if (B * S == 0) return KVQ_OK;
    if (!kv->data || !gamma->data || !cos->data || !sin->data || !index->data || !k_cache->data ||
        !ckv_cache->data || (kc.scale_n && !kc.scale) || (cc.scale_n && !cc.scale) ||
        (kc.offset_n && !kc.offset) || (cc.offset_n && !cc.offset))
        return KVQ_ERR_NULL;

    RmsRopeArgs a;
    a.kv = static_cast<const uint16_t*>(kv->data);
    a.kv_f16 = kv->dtype == KVQ_F16;
    a.B = B;
    a.S = S;
    a.D = (int32_t)D;
    a.Dv = (int32_t)Dv;
    a.Dk = (int32_t)Dk;
    a.gamma = static_cast<const uint16_t*>(gamma->data);
    a.cos = static_cast<const uint16_t*>(cos->data);
    a.sin = static_cast<const uint16_t*>(sin->data);
    a.index = index->data;
    a.index_i64 = index->dtype == KVQ_I64;
    a.cache_mode = cache_mode;
    a.k = kc;
    a.ckv = cc;
    a.eps = epsilon;
    const int64_t warps_per_block = RR_THREADS / 32;
    const int64_t need = (B * S + warps_per_block - 1) / warps_per_block;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool vec = reinterpret_cast<uintptr_t>(kv->data) % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(gamma->data) % 16 == 0 && D % 8 == 0 && Dv % 8 == 0;
    const int64_t nch = Dv / 8;
    // the register-chunk kernels stage an int8 ckv cache's parameters in shared memory
    a.ckv_stage = vec && nch <= 128 && cc.dt == CDT_I8;
    a.inv_dv = (Dv & (Dv - 1)) == 0 ? 1.0f / (float)Dv : 0.0f;     // exact: a power of two
    const size_t smem = a.ckv_stage ? (size_t)3 * Dv * sizeof(float) : 0;
    auto run = [&](auto kernel, size_t sm) {
        return launched(launch(kernel, (unsigned)persistent_grid(kernel, RR_THREADS, need, sm), RR_THREADS, sm, s, a));
    };
    // the lean kernel: Dv of 256, 512 or 1024, Dk = 64, one index entry per
    // token, fewer than 2^31 tokens and slots, 32-bit block strides, and cache
    // rows aligned for its whole-chunk stores (16 bytes for a 16-bit ckv
    // cache, 8 for FP8 codes; 2 for a 16-bit k cache)
    auto rows_aligned = [](const PagedRows& r, int64_t q) {
        return reinterpret_cast<uintptr_t>(r.base) % q == 0 && r.row_bytes % q == 0 && r.block_stride % q == 0;
    };
    const bool k16 = kc.dt == CDT_BF16 || kc.dt == CDT_F16;
    const bool lean = vec && (Dv == 256 || Dv == 512 || Dv == 1024) && Dk == 64 &&
                      (cache_mode == 1 || cache_mode == 2) && B * S < (1LL << 31) &&
                      kc.rows.num_slots < (1LL << 31) && cc.rows.block_stride < (1LL << 32) &&
                      kc.rows.block_stride < (1LL << 32) && bs * cc.rows.row_bytes < (1LL << 32) &&
                      bs * kc.rows.row_bytes < (1LL << 32) &&
                      rows_aligned(cc.rows, cc.dt == CDT_BF16 || cc.dt == CDT_F16 ? 16 : 8) &&
                      (!k16 || rows_aligned(kc.rows, 2));
    if (lean) {
        const int lck = cc.dt == CDT_E4M3 ? 1 : (cc.dt == CDT_E5M2 ? 3 : (cc.dt == CDT_I8 ? 2 : 0));
        const size_t lsm = (size_t)Dv * sizeof(float) * (lck == 2 ? 4 : 1);
#define KVQ_RR_LEAN(N, C) \
    return a.kv_f16 ? run(rmsnorm_rope_lean_kernel<N, C, true>, lsm) : run(rmsnorm_rope_lean_kernel<N, C, false>, lsm)
#define KVQ_RR_LEAN_N(N)                     \
    switch (lck) {                           \
        case 0: KVQ_RR_LEAN(N, 0);           \
        case 1: KVQ_RR_LEAN(N, 1);           \
        case 2: KVQ_RR_LEAN(N, 2);           \
        default: KVQ_RR_LEAN(N, 3);          \
    }
        if (Dv == 256) KVQ_RR_LEAN_N(1);
        if (Dv == 512) KVQ_RR_LEAN_N(2);
        KVQ_RR_LEAN_N(4);
#undef KVQ_RR_LEAN_N
#undef KVQ_RR_LEAN
    }
    const int ck = ckv_class(cc.dt);
#define KVQ_RR_CK(N)                                                                           \
    return ck == 0 ? run(rmsnorm_rope_kernel<N, 0>, smem)                                      \
                   : (ck == 1 ? run(rmsnorm_rope_kernel<N, 1>, smem) : run(rmsnorm_rope_kernel<N, 2>, smem))
    if (vec && nch <= 32) KVQ_RR_CK(1);
    if (vec && nch <= 64) KVQ_RR_CK(2);
    if (vec && nch <= 128) KVQ_RR_CK(4);
#undef KVQ_RR_CK
    return run(rmsnorm_rope_kernel<0>, (size_t)0);
}

// ---------------------------------------------------------------------------
kvq_status kvq_dequant_rope_quant_kvcache(const kvq_tensor* x, const kvq_tensor* cos, const kvq_tensor* sin,
                                          kvq_tensor* k_cache, kvq_tensor* v_cache, const kvq_tensor* indices,
                                          const kvq_tensor* scale_k, const kvq_tensor* scale_v,
                                          const kvq_tensor* offset_k, const kvq_tensor* offset_v,
                                          const kvq_tensor* weight_scale, const kvq_tensor* activation_scale,
                                          const kvq_tensor* bias, const int64_t* size_splits, int32_t n_splits,
                                          int32_t quant_mode, int32_t layout, int32_t kv_output,
                                          int32_t cache_mode, kvq_tensor* q_out, kvq_tensor* k_out,
                                          kvq_tensor* v_out, kvq_stream stream) {
    Trace trace("kvq_dequant_rope_quant_kvcache");
    if (!x || !cos || !sin || !k_cache || !v_cache || !indices || !scale_k || !scale_v || !q_out || !size_splits)
        return KVQ_ERR_NULL;
    if (!valid_desc(x) || !valid_desc(cos) || !valid_desc(sin) || !valid_desc(k_cache) || !valid_desc(v_cache) ||
        !valid_desc(indices) || !valid_desc(scale_k) || !valid_desc(scale_v) || !valid_desc(q_out))
        return KVQ_ERR_DTYPE;
    if (quant_mode != 0 || layout != 0 || (cache_mode != 0 && cache_mode != 1) || n_splits != 3)
        return KVQ_ERR_ATTR;
    if (x->dtype != KVQ_I32 && x->dtype != KVQ_BF16 && x->dtype != KVQ_F16) return KVQ_ERR_DTYPE;
    if (cos->dtype != KVQ_BF16 && cos->dtype != KVQ_F16) return KVQ_ERR_DTYPE;
    if (sin->dtype != cos->dtype || q_out->dtype != cos->dtype) return KVQ_ERR_DTYPE;
    if (x->dtype != KVQ_I32 && x->dtype != cos->dtype) return KVQ_ERR_DTYPE;
    if (x->ndim != 2 && x->ndim != 3) return KVQ_ERR_NDIM;
    if (k_cache->ndim != 4 || v_cache->ndim != 4) return KVQ_ERR_NDIM;
    if (k_cache->dtype != KVQ_I8 || v_cache->dtype != KVQ_I8) return KVQ_ERR_DTYPE;
    const int64_t B = x->shape[0];
    const int64_t S = x->ndim == 3 ? x->shape[1] : 1;
    const int64_t H = x->shape[x->ndim - 1];
    if (size_splits[1] != size_splits[2]) return KVQ_ERR_ATTR;
    const int64_t D = k_cache->shape[3];
    if (D <= 0 || D % 16 != 0) return KVQ_ERR_SHAPE;
    if (size_splits[0] <= 0 || size_splits[1] <= 0 || size_splits[0] % D || size_splits[1] % D) return KVQ_ERR_SHAPE;
    if (size_splits[0] + size_splits[1] + size_splits[2] != H) return KVQ_ERR_SHAPE;
    if (H > 4096 || H % 64 != 0) return KVQ_ERR_SHAPE;
    const int64_t Nq = size_splits[0] / D, Nkv = size_splits[1] / D;
    if (k_cache->shape[2] != Nkv) return KVQ_ERR_SHAPE;
    for (int i = 0; i < 4; ++i)
        if (k_cache->shape[i] != v_cache->shape[i]) return KVQ_ERR_SHAPE;
    PagedRows kr, vr;
    int64_t hd;
    kvq_status st = paged_from(k_cache, Nkv, &kr, &hd);
    if (st != KVQ_OK) return st;
    st = paged_from(v_cache, Nkv, &vr, &hd);
    if (st != KVQ_OK) return st;
    if (!contiguous(x) || !contiguous(cos) || !contiguous(sin) || !contiguous(indices) || !contiguous(q_out))
        return KVQ_ERR_LAYOUT;
    if (numel(cos) != B * S * D || numel(sin) != B * S * D) return KVQ_ERR_SHAPE;
    if (numel(q_out) != B * S * Nq * D) return KVQ_ERR_SHAPE;
    if (!is_index_dtype(indices->dtype)) return KVQ_ERR_DTYPE;
    if (numel(indices) != (cache_mode == 1 ? B * S : B)) return KVQ_ERR_SHAPE;
    if (cache_mode == 0 && (k_cache->shape[0] < B || k_cache->shape[1] < S)) return KVQ_ERR_SHAPE;
    const float *sk = nullptr, *sv = nullptr, *ok = nullptr, *ov = nullptr, *ws = nullptr, *as = nullptr;
    auto f32param = [](const kvq_tensor* p, int64_t n, bool required, const float** out) -> kvq_status {
        if (!p) return required ? KVQ_ERR_NULL : KVQ_OK;
        if (!valid_desc(p) || p->dtype != KVQ_F32) return KVQ_ERR_DTYPE;
        if (numel(p) != n) return KVQ_ERR_SHAPE;
        if (!contiguous(p)) return KVQ_ERR_LAYOUT;
        *out = static_cast<const float*>(p->data);
        return KVQ_OK;
    };
    const bool dq = x->dtype == KVQ_I32;
    if ((st = f32param(scale_k, Nkv * D, true, &sk)) != KVQ_OK) return st;
    if ((st = f32param(scale_v, Nkv * D, true, &sv)) != KVQ_OK) return st;
    if ((st = f32param(offset_k, Nkv * D, false, &ok)) != KVQ_OK) return st;
    if ((st = f32param(offset_v, Nkv * D, false, &ov)) != KVQ_OK) return st;
    if (dq) {
        if ((st = f32param(weight_scale, H, true, &ws)) != KVQ_OK) return st;
        if ((st = f32param(activation_scale, B * S, false, &as)) != KVQ_OK) return st;
    }
    int32_t bias_kind = 0;
    const void* bias_ptr = nullptr;
    if (dq && bias) {
        if (!valid_desc(bias)) return KVQ_ERR_DTYPE;
        switch (bias->dtype) {
            case KVQ_F32: bias_kind = 0; break;
            case KVQ_F16: bias_kind = 1; break;
            case KVQ_BF16: bias_kind = 2; break;
            case KVQ_I32: bias_kind = 3; break;
            default: return KVQ_ERR_DTYPE;
        }
        if (numel(bias) != H) return KVQ_ERR_SHAPE;
        if (!contiguous(bias)) return KVQ_ERR_LAYOUT;
        bias_ptr = bias->data;
    }
    uint16_t *kop = nullptr, *vop = nullptr;
    if (kv_output) {
        if (!k_out || !v_out) return KVQ_ERR_NULL;
        if (!valid_desc(k_out) || !valid_desc(v_out)) return KVQ_ERR_DTYPE;
        if (k_out->dtype != cos->dtype || v_out->dtype != cos->dtype) return KVQ_ERR_DTYPE;
        if (numel(k_out) != B * S * Nkv * D || numel(v_out) != B * S * Nkv * D) return KVQ_ERR_SHAPE;
        if (!contiguous(k_out) || !contiguous(v_out)) return KVQ_ERR_LAYOUT;
        kop = static_cast<uint16_t*>(k_out->data);
        vop = static_cast<uint16_t*>(v_out->data);
    }
    if (B * S == 0) return KVQ_OK;
    if (!x->data || !cos->data || !sin->data || !indices->data || !q_out->data || !k_cache->data || !v_cache->data ||
        (kv_output && (!kop || !vop)) || !sk || !sv || (offset_k && !ok) || (offset_v && !ov) || (dq && !ws) ||
        (dq && activation_scale && !as) || (dq && bias && !bias_ptr))
        return KVQ_ERR_NULL;

    DrqArgs a;
    a.x = x->data;
    a.x_kind = dq ? 0 : (x->dtype == KVQ_BF16 ? 1 : 2);
    a.x_vec = reinterpret_cast<uintptr_t>(x->data) % 16 == 0;
    a.tps = 0;
    a.stages = 0;
    a.B = B;
    a.S = S;
    a.H = H;
    a.cos = static_cast<const uint16_t*>(cos->data);
    a.sin = static_cast<const uint16_t*>(sin->data);
    a.cos_f16 = cos->dtype == KVQ_F16;
    a.kc = kr;
    a.vc = vr;
    a.indices = indices->data;
    a.indices_i64 = indices->dtype == KVQ_I64;
    a.cache_mode = cache_mode;
    a.scale_k = sk;
    a.scale_v = sv;
    a.offset_k = ok;
    a.offset_v = ov;
    a.weight_scale = ws;
    a.activation_scale = as;
    a.bias = bias_ptr;
    a.bias_kind = bias_kind;
    {
        auto al = [](const void* p) { return p == nullptr || reinterpret_cast<uintptr_t>(p) % 16 == 0; };
        a.params_vec = al(sk) && al(sv) && al(ok) && al(ov) && al(ws) && (bias_kind != 0 || al(bias_ptr));
        auto al8 = [](const void* p) { return p == nullptr || reinterpret_cast<uintptr_t>(p) % 8 == 0; };
        a.out_vec8 = al8(q_out->data) && al8(kop) && al8(vop);
        auto r4 = [](const PagedRows& r) {
            return reinterpret_cast<uintptr_t>(r.base) % 4 == 0 && r.row_bytes % 4 == 0 && r.block_stride % 4 == 0;
        };
        a.rows_vec4 = r4(kr) && r4(vr);
    }
    a.Nq = (int32_t)Nq;
    a.Nkv = (int32_t)Nkv;
    a.D = (int32_t)D;
    a.q_out = static_cast<uint16_t*>(q_out->data);
    a.k_out = kop;
    a.v_out = vop;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t need = B * S;
    const int xb = dq ? 4 : 2;
    const bool aligned = reinterpret_cast<uintptr_t>(x->data) % 16 == 0 &&
                         reinterpret_cast<uintptr_t>(cos->data) % 16 == 0 &&
                         reinterpret_cast<uintptr_t>(sin->data) % 16 == 0 && (D * 2) % 16 == 0;
    const size_t prm = dt_param_bytes(H, Nkv * D, dq);
    if (aligned && D % 8 == 0 && D <= 256 && prm <= 64 * 1024) {
        // pipelined kernel: token rows, cos and sin arrive in shared memory by
        // bulk copy; TPS tokens per stage (a divisor of the consumer warps, x
        // span at most 32 KB), as many stages (2..4) as keep two CTAs on an SM
        int tps = 1;
        while (tps < DT_CONSUMERS && 2 * tps * H * xb <= 32768) tps *= 2;     // 2, 4 or 8 (H <= 4096)
        a.tps = tps;
        auto dt_smem = [&](int stages) {
            return (size_t)dt_header_bytes(stages, tps) + prm + (size_t)stages * dt_stage_bytes(tps, H, xb, (int)D);
        };
        a.stages = 4;
        while (a.stages > 2 && dt_smem(a.stages) > 112 * 1024) --a.stages;
        const size_t smem = dt_smem(a.stages);
        const int64_t tiles = (need + a.tps - 1) / a.tps;
        const bool f16 = a.cos_f16 != 0;
        if (a.x_kind == 0) return launched(f16 ? launch_drq_ring<0, true>(a, tiles, smem, s)
                                               : launch_drq_ring<0, false>(a, tiles, smem, s));
        if (a.x_kind == 1) return launched(launch_drq_ring<1, false>(a, tiles, smem, s));
        return launched(launch_drq_ring<2, true>(a, tiles, smem, s));
    }
    // every other shape and alignment: one CTA per token
    return launched(launch(dequant_rope_quant_general_kernel,
                           (unsigned)persistent_grid(dequant_rope_quant_general_kernel, DG_THREADS, need),
                           DG_THREADS, 0, s, a));
}

// ---------------------------------------------------------------------------
kvq_status kvq_get_error(kvq_stream stream, uint32_t* fault_bits) {
    if (!fault_bits) return KVQ_ERR_NULL;
    *fault_bits = 0u;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // one device-side atomic exchange reads and clears the word, so a bit
    // raised by a kernel on another stream is either returned by this call or
    // left for the next one; concurrent callers take different snapshot slots
    static std::atomic<uint32_t> ticket{0};
    const uint32_t slot = ticket.fetch_add(1u, std::memory_order_relaxed) % FAULT_SNAPSHOTS;
    unsigned int h = 0u;
    // a plain launch (no programmatic serialization): the exchange runs after
    // every earlier kernel of the stream has completed
    uint32_t slot_arg = slot;
    void* args[] = {&slot_arg};
    if (cudaLaunchKernel(reinterpret_cast<const void*>(fault_exchange_kernel), dim3(1), dim3(1), args, 0, s) !=
        cudaSuccess)
        return KVQ_ERR_CUDA;
    if (cudaMemcpyFromSymbolAsync(&h, g_fault_snapshot, sizeof(h), slot * sizeof(h), cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return KVQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return KVQ_ERR_CUDA;
    *fault_bits = h;
    return KVQ_OK;
}

// ---------------------------------------------------------------------------
namespace {

// cuTensorMapEncodeTiled through the runtime's driver entry point (the
// library links the CUDA runtime statically and never links the driver
// library itself)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Tensor map of a row-major bf16 matrix [rows, cols] (row pitch `pitch`
// elements) read in boxes of box_rows x 64 columns with the 128-byte swizzle;
// rows past the end read as zero.
bool bf16_tile_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t pitch, uint32_t box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(pitch * 2)};
    const cuuint32_t box[2] = {(cuuint32_t)CP_BK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The C4A weights [2 D, H] bf16 (rows [0, D) the a half, [D, 2 D) the b half)
// as a 4-D tensor {k: H, row: 8, half: 2, block: D / 8} with 128-byte swizzled
// boxes {64, 8, 2, 8}: one box holds 64 channels' a and b rows, interleaved in
// blocks of 8 rows (a then b) along k slices of 64.
bool bf16_pair_map(CUtensorMap* m, const void* base, int64_t D, int64_t H) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)H, 8, 2, (cuuint64_t)(D / 8)};
    const cuuint64_t strides[3] = {(cuuint64_t)(H * 2), (cuuint64_t)(D * H * 2), (cuuint64_t)(8 * H * 2)};
    const cuuint32_t box[4] = {(cuuint32_t)CP_BK, 8, 2, 8};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

kvq_status kvq_compressor(const kvq_tensor* x, const kvq_tensor* w_kv, const kvq_tensor* w_gate,
                          const kvq_tensor* ape, kvq_tensor* cmp_kv, int32_t cmp_ratio, kvq_stream stream) {
    Trace trace("kvq_compressor");
    if (!x || !w_kv || !w_gate || !ape || !cmp_kv) return KVQ_ERR_NULL;
    if (!valid_desc(x) || !valid_desc(w_kv) || !valid_desc(w_gate) || !valid_desc(ape) || !valid_desc(cmp_kv))
        return KVQ_ERR_DTYPE;
    if (x->dtype != KVQ_BF16 || w_kv->dtype != KVQ_BF16 || w_gate->dtype != KVQ_BF16 || cmp_kv->dtype != KVQ_BF16 ||
        ape->dtype != KVQ_F32)
        return KVQ_ERR_DTYPE;
    if (cmp_ratio < 2 || cmp_ratio > 128 || (cmp_ratio & (cmp_ratio - 1)) != 0) return KVQ_ERR_ATTR;
    if (x->ndim < 1 || w_kv->ndim != 2 || w_gate->ndim != 2 || ape->ndim != 2 || cmp_kv->ndim != 2)
        return KVQ_ERR_NDIM;
    const int64_t H = x->shape[x->ndim - 1];
    const int64_t T = numel_leading(x);
    const int64_t D = cmp_kv->shape[1];
    if (H < 1024 || H > 10240 || H % 512 != 0) return KVQ_ERR_SHAPE;
    if (D != 128 && D != 512) return KVQ_ERR_SHAPE;
    // coff from the weights: [D, H] (the C128A form) or [2 D, H] (C4A / C4Li,
    // cmp_ratio 4)
    const int64_t coff = w_kv->shape[0] == D ? 1 : (w_kv->shape[0] == 2 * D ? 2 : 0);
    if (coff == 0) return KVQ_ERR_SHAPE;
    if (coff == 2 && cmp_ratio != 4) return KVQ_ERR_ATTR;
    if (w_kv->shape[1] != H || w_gate->shape[0] != coff * D || w_gate->shape[1] != H) return KVQ_ERR_SHAPE;
    if (ape->shape[0] != cmp_ratio || ape->shape[1] != coff * D) return KVQ_ERR_SHAPE;
    if (T % cmp_ratio != 0) return KVQ_ERR_SHAPE;
    if (cmp_kv->shape[0] != T / cmp_ratio) return KVQ_ERR_SHAPE;
    if (T > (int64_t)0x7fffffff - CP_BN) return KVQ_ERR_SHAPE;          // TMA coordinates are 32-bit
    if (!contiguous(x) || !contiguous(w_kv) || !contiguous(w_gate) || !contiguous(ape) || !contiguous(cmp_kv))
        return KVQ_ERR_LAYOUT;
    if (T == 0) return KVQ_OK;
    if (!x->data || !w_kv->data || !w_gate->data || !ape->data || !cmp_kv->data) return KVQ_ERR_NULL;
    auto a16 = [](const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; };
    if (!a16(x->data) || !a16(w_kv->data) || !a16(w_gate->data)) return KVQ_ERR_LAYOUT;   // TMA base alignment

    // token tiles of 256, or of 128 when 256-token tiles would fill at most
    // half of the SMs (twice the tiles for a small batch).  C128A: 128 channels
    // and BN tokens per tile; C4A: 64 channel pairs (a and b) and BN tokens,
    // consecutive tiles BN - 4 tokens apart (BN / 4 - 1 groups each)
    const int64_t n_ch = coff == 1 ? D / CP_BM : D / (CP_BM / 2);
    auto tok_tiles = [&](int bn) {
        return coff == 1 ? (T + bn - 1) / bn : (T / 4 + bn / 4 - 2) / (bn / 4 - 1);
    };
    const int bn = 2 * tok_tiles(256) * n_ch <= (int64_t)sm_count() ? 128 : 256;
    CUtensorMap mx, mk, mg;
    if (!bf16_tile_map(&mx, x->data, T, H, H, (uint32_t)bn)) return KVQ_ERR_CUDA;
    if (coff == 1 ? !bf16_tile_map(&mk, w_kv->data, D, H, H, CP_BM) || !bf16_tile_map(&mg, w_gate->data, D, H, H, CP_BM)
                  : !bf16_pair_map(&mk, w_kv->data, D, H) || !bf16_pair_map(&mg, w_gate->data, D, H))
        return KVQ_ERR_CUDA;
    CompressorArgs a;
    a.T = T;
    a.H = (int32_t)H;
    a.D = (int32_t)D;
    a.n_ch_tiles = (int32_t)n_ch;
    a.n_tok_tiles = tok_tiles(bn);
    a.ape = static_cast<const float*>(ape->data);
    a.out = static_cast<uint16_t*>(cmp_kv->data);
    const int64_t tiles = a.n_tok_tiles * a.n_ch_tiles;
    const size_t smem = cp_smem_bytes(bn);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    auto run = [&](auto kernel) {
        return launched(launch(kernel, (unsigned)persistent_grid(kernel, CP_THREADS, tiles, smem), CP_THREADS, smem,
                               s, mx, mk, mg, a));
    };
#define KVQ_CP_RATIOS(BN)                                 \
    switch (cmp_ratio) {                                  \
        case 2: return run(compressor_kernel<2, BN>);     \
        case 4: return run(compressor_kernel<4, BN>);     \
        case 8: return run(compressor_kernel<8, BN>);     \
        case 16: return run(compressor_kernel<16, BN>);   \
        case 32: return run(compressor_kernel<32, BN>);   \
        case 64: return run(compressor_kernel<64, BN>);   \
        default: return run(compressor_kernel<128, BN>);  \
    }
    if (coff == 2) return bn == 128 ? run(compressor_kernel<4, 128, 2>) : run(compressor_kernel<4, 256, 2>);
    if (bn == 128) KVQ_CP_RATIOS(128);
    KVQ_CP_RATIOS(256);
#undef KVQ_CP_RATIOS
}

// ---------------------------------------------------------------------------
kvq_status kvq_scatter_rows(const kvq_tensor* x, const kvq_tensor* slot_mapping, kvq_tensor* cache,
                            int64_t out_bytes, kvq_stream stream) {
    Trace trace("kvq_scatter_rows");
    if (!x || !slot_mapping || !cache) return KVQ_ERR_NULL;
    if (!valid_desc(x) || !valid_desc(slot_mapping) || !valid_desc(cache)) return KVQ_ERR_DTYPE;
    if (x->ndim < 1) return KVQ_ERR_NDIM;
    int64_t T, rs;
    if (!flatten_rows(x, &T, &rs)) return KVQ_ERR_LAYOUT;
    const int64_t eb = elem_bytes(x->dtype);
    const int64_t in_bytes = x->shape[x->ndim - 1] * eb;
    if (in_bytes % 16 != 0 || in_bytes < 16 || in_bytes > SB_MAX_ROW_BYTES) return KVQ_ERR_SHAPE;
    if (out_bytes < 16 || out_bytes % 16 != 0 || out_bytes > in_bytes) return KVQ_ERR_ATTR;
    if (!is_index_dtype(slot_mapping->dtype)) return KVQ_ERR_DTYPE;
    if (numel(slot_mapping) != T) return KVQ_ERR_SHAPE;
    if (!contiguous(slot_mapping)) return KVQ_ERR_LAYOUT;
    if (cache->dtype != KVQ_U8 && cache->dtype != KVQ_I8) return KVQ_ERR_DTYPE;
    if (cache->ndim != 4) return KVQ_ERR_NDIM;
    if (cache->shape[2] != 1) return KVQ_ERR_SHAPE;
    PagedRows rows;
    int64_t head_dim;
    kvq_status st = paged_from(cache, 1, &rows, &head_dim);
    if (st != KVQ_OK) return st;
    if (head_dim < out_bytes) return KVQ_ERR_CAPACITY;
    if (T == 0) return KVQ_OK;
    if (!x->data || !slot_mapping->data || !cache->data) return KVQ_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(x->data) % 16 != 0 || (rs * eb) % 16 != 0 ||
        reinterpret_cast<uintptr_t>(cache->data) % 16 != 0 || rows.row_bytes % 16 != 0 ||
        rows.block_stride % 16 != 0)
        return KVQ_ERR_LAYOUT;
    ScatterCopyArgs a;
    a.x = static_cast<const uint8_t*>(x->data);
    a.x_row_bytes = rs * eb;
    a.T = T;
    a.slots = slot_mapping->data;
    a.slots_i64 = slot_mapping->dtype == KVQ_I64;
    a.cache = rows;
    a.in_bytes = (int32_t)in_bytes;
    a.out_bytes = (int32_t)out_bytes;
    const size_t smem = sb_smem_bytes((int)in_bytes);
    const int64_t tiles = (T + SB_ROWS - 1) / SB_ROWS;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return launched(launch(scatter_bulk_kernel, (unsigned)persistent_grid(scatter_bulk_kernel, SB_THREADS, tiles, smem),
                           SB_THREADS, smem, s, a));
}

kvq_status kvq_convert(int32_t fmt, const float* in, int64_t n, void* out, kvq_stream stream) {
    if (fmt < 0 || fmt > 5) return KVQ_ERR_ATTR;
    if (n < 0) return KVQ_ERR_SHAPE;
    if (n == 0) return KVQ_OK;
    if (!in || !out) return KVQ_ERR_NULL;
    const int64_t need = (n + 255) / 256;
    return launched(launch(convert_kernel, (unsigned)persistent_grid(convert_kernel, 256, need), 256, 0,
                           reinterpret_cast<cudaStream_t>(stream), fmt, in, n, static_cast<uint8_t*>(out)));
}

}  // extern "C"
