/*
 * kvq_oracle.c -- plain, slow CPU oracle for the per-token KV-cache epilogue.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent statement of what
 * the four epilogue operations compute.  Only the test suite, the smoke check
 * and the benchmark's CPU-baseline leg may load it.  It shares no source with
 * the CUDA library (kv_cache_quantize_b200/csrc) and includes none of its
 * headers; the CUDA library never calls it.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (see oracle/build.py).  -ffp-contract=off keeps every a*b+c as two IEEE
 * binary32 roundings, so each expression below is evaluated in exactly the
 * order it is written.  On x86-64 float arithmetic is SSE binary32 with
 * round-to-nearest-even and no flush-to-zero, FLT_EVAL_METHOD == 0.
 *
 * Sources (page title, section):
 *   [EPI]  aclnnKvCompressEpilog            -- 接口功能 / 计算公式 / 约束说明
 *   [RMS]  aclnnKvRmsNormRopeCache          -- 计算公式 (interleaveRope, rmsNorm) / 约束说明
 *   [IDX]  indexer_quant_cache (torch_npu)  -- 接口功能 / 约束说明
 *   [DRQ]  aclnnDequantRopeQuantKvcache 算子深度解析 (blog)
 *          -- 计算步骤公式, 两种 KV Cache 更新模式, 约束说明, Kernel 实现要点
 *
 * Where the pages leave a step open the reading used here is stated next to
 * the step; every such reading is also listed in the design notes.
 *
 * Pinning: every function here is checked by tests/test_oracle_*.py against
 * values fixed by the pages or by mathematics (printed worked examples,
 * format definitions, brute-force nearest search, exact rational arithmetic,
 * library routines, invariants).  The conventions marked "parity unpinned"
 * below (packed-row segment order, FP4 nibble order, padding bytes,
 * quant_mode numbering of the indexer beyond mode 0) have no such pin.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Fault bits reported for data the pages declare invalid (bad slot index). */
#define KVQO_FAULT_SLOT_RANGE 0x1u

/* Status codes of the oracle (parameter problems only; the oracle is not  */
/* the validator, it refuses what it cannot compute).                      */
#define KVQO_OK 0
#define KVQO_EINVAL 1

/* ------------------------------------------------------------------------ */
/* Number formats, written from their definitions.                          */
/*                                                                          */
/* A binary floating-point format with E exponent bits, M fraction bits and */
/* exponent bias B represents                                               */
/*   normal     (-1)^s * (1 + f/2^M) * 2^(e - B),   1 <= e                  */
/*   subnormal  (-1)^s * (f/2^M) * 2^(1 - B),        e == 0                 */
/* FP8 E4M3FN: E=4 M=3 B=7,   no infinities, S.1111.111 is NaN, max 448.    */
/* FP8 E5M2:   E=5 M=2 B=15,  IEEE-style inf/NaN, max finite 57344.         */
/* FP4 E2M1:   E=2 M=1 B=1,   no inf/NaN, values {0,.5,1,1.5,2,3,4,6}.      */
/* bfloat16:   E=8 M=7 B=127; IEEE binary16: E=5 M=10 B=15.                 */
/* E8M0 (scale): 8-bit unsigned exponent b, value 2^(b-127), 0xFF is NaN.   */
/* ------------------------------------------------------------------------ */

typedef struct {
    int ebits;
    int mbits;
    int bias;
    double maxval;   /* largest finite magnitude */
    int has_inf;     /* overflow without saturation goes to infinity */
    uint32_t nan_code;
} kvqo_fmt;

static const kvqo_fmt FMT_E4M3 = {4, 3, 7, 448.0, 0, 0x7Fu};
static const kvqo_fmt FMT_E5M2 = {5, 2, 15, 57344.0, 1, 0x7Fu};
static const kvqo_fmt FMT_E2M1 = {2, 1, 1, 6.0, 0, 0x7u};
/* (2 - 2^-7) * 2^127 and (2 - 2^-10) * 2^15 */
static const kvqo_fmt FMT_BF16 = {8, 7, 127, 3.3895313892515355e38, 1, 0x7FC0u};
static const kvqo_fmt FMT_F16 = {5, 10, 15, 65504.0, 1, 0x7E00u};

/* Round a finite magnitude a >= 0 to the format's grid: the nearest value  */
/* with an M-bit fraction, ties to the even significand.  Below the         */
/* smallest normal binade every value shares that binade's quantum (the     */
/* subnormal spacing).  a is a binary32 value, so a, the quantum and the    */
/* quotient are exact in binary64; nearbyint rounds half to even in the     */
/* default rounding mode.                                                   */
static double grid_round(double a, int mbits, int emin)
{
    if (a == 0.0) return 0.0;
    int e2;
    frexp(a, &e2);           /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;          /* a in [2^E, 2^(E+1)) */
    if (E < emin) E = emin;
    double quantum = ldexp(1.0, E - mbits);
    double k = a / quantum;  /* exact */
    return nearbyint(k) * quantum;
}

/* Bit pattern of a magnitude r that lies exactly on the format's grid. */
static uint32_t pack_magnitude(const kvqo_fmt* f, double r)
{
    if (r == 0.0) return 0u;
    int emin = 1 - f->bias;
    int e2;
    frexp(r, &e2);
    int E = e2 - 1;
    if (E < emin) {
        double frac = r / ldexp(1.0, emin - f->mbits);
        return (uint32_t)frac;                              /* exponent field 0 */
    }
    double frac = r / ldexp(1.0, E - f->mbits) - ldexp(1.0, f->mbits);
    return ((uint32_t)(E + f->bias) << f->mbits) | (uint32_t)frac;
}

/* Encode a binary32 value: round to nearest, ties to even.  With saturate */
/* set, results beyond the largest finite value are clamped to it (the     */
/* "satfinite" behaviour); the sign is kept, including for -0.             */
static uint32_t encode_rn(const kvqo_fmt* f, float v, int saturate)
{
    uint32_t sign = signbit(v) ? 1u : 0u;
    uint32_t sign_bit = sign << (f->ebits + f->mbits);
    if (isnan(v)) return f->nan_code;
    double a = fabs((double)v);
    double r;
    if (isinf(a)) {
        r = INFINITY;
    } else {
        r = grid_round(a, f->mbits, 1 - f->bias);
    }
    if (r > f->maxval) {
        if (saturate || !f->has_inf) {
            r = f->maxval;
        } else {
            uint32_t inf = ((1u << f->ebits) - 1u) << f->mbits;
            return sign_bit | inf;
        }
    }
    return sign_bit | pack_magnitude(f, r);
}

static float decode_bits(const kvqo_fmt* f, uint32_t code)
{
    uint32_t mmask = (1u << f->mbits) - 1u;
    uint32_t emask = (1u << f->ebits) - 1u;
    uint32_t s = (code >> (f->ebits + f->mbits)) & 1u;
    uint32_t e = (code >> f->mbits) & emask;
    uint32_t m = code & mmask;
    double v;
    if (e == 0) {
        v = ldexp((double)m, 1 - f->bias - f->mbits);
    } else if (f->has_inf && e == emask) {
        v = (m == 0) ? INFINITY : NAN;
    } else if (f == &FMT_E4M3 && e == emask && m == mmask) {
        v = NAN;                                  /* S.1111.111 */
    } else {
        v = ldexp((double)(m + (1u << f->mbits)), (int)e - f->bias - f->mbits);
    }
    return (float)(s ? -v : v);
}

static float bf16_to_f32(uint16_t h) { return decode_bits(&FMT_BF16, h); }
static float f16_to_f32(uint16_t h) { return decode_bits(&FMT_F16, h); }
static uint16_t f32_to_bf16(float v) { return (uint16_t)encode_rn(&FMT_BF16, v, 0); }
static uint16_t f32_to_f16(float v) { return (uint16_t)encode_rn(&FMT_F16, v, 0); }
static uint8_t enc_e4m3(float v) { return (uint8_t)encode_rn(&FMT_E4M3, v, 1); }
static uint8_t enc_e5m2(float v) { return (uint8_t)encode_rn(&FMT_E5M2, v, 1); }
static uint8_t enc_e2m1(float v) { return (uint8_t)encode_rn(&FMT_E2M1, v, 1); }

/* E8M0 scale rounded up to a power of two: the smallest b in [0, 254] with */
/* 2^(b-127) >= q.  q == 0 gives b = 0.  Written as the search it defines.  */
static uint8_t e8m0_ceil(float q)
{
    for (int b = 0; b <= 254; ++b) {
        if (ldexp(1.0, b - 127) >= (double)q) return (uint8_t)b;
    }
    return 254;
}

static float pow2f(int k) { return ldexpf(1.0f, k); }

/* Static int8 quantisation of [DRQ] Kernel 实现要点 (量化): Cast with RINT */
/* to int16, then to half, then to int8.  Every stage is monotone and exact */
/* on [-128, 127]; with saturating casts the chain is clamp(rint_even(v)). */
/* NaN maps to 0 (the inputs of the pages are finite).                      */
static int8_t int8_static(float v)
{
    if (isnan(v)) return 0;
    float r = nearbyintf(v);
    if (r > 127.0f) return 127;
    if (r < -128.0f) return -128;
    return (int8_t)r;
}

/* ------------------------------------------------------------------------ */
/* Exported codec entry points (used by the oracle's own tests).            */
/* fmt: 0 E4M3, 1 E5M2, 2 E2M1, 3 bf16, 4 f16                               */
/* ------------------------------------------------------------------------ */
static const kvqo_fmt* fmt_by_id(int id)
{
    switch (id) {
        case 0: return &FMT_E4M3;
        case 1: return &FMT_E5M2;
        case 2: return &FMT_E2M1;
        case 3: return &FMT_BF16;
        case 4: return &FMT_F16;
        default: return NULL;
    }
}

int kvqo_encode_array(int fmt_id, const float* v, int64_t n, int saturate, uint32_t* out)
{
    const kvqo_fmt* f = fmt_by_id(fmt_id);
    if (!f) return KVQO_EINVAL;
    for (int64_t i = 0; i < n; ++i) out[i] = encode_rn(f, v[i], saturate);
    return KVQO_OK;
}

int kvqo_decode_array(int fmt_id, const uint32_t* code, int64_t n, float* out)
{
    const kvqo_fmt* f = fmt_by_id(fmt_id);
    if (!f) return KVQO_EINVAL;
    for (int64_t i = 0; i < n; ++i) out[i] = decode_bits(f, code[i]);
    return KVQO_OK;
}

int kvqo_e8m0_ceil_array(const float* q, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = e8m0_ceil(q[i]);
    return KVQO_OK;
}

int kvqo_int8_static_array(const float* v, int64_t n, int8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = int8_static(v[i]);
    return KVQO_OK;
}

/* ------------------------------------------------------------------------ */
/* Paged cache geometry.  A cache [blockNum, blockSize, 1, headDim] holds    */
/* num_slots = blockNum * blockSize rows; slot s lives in block             */
/* s / blockSize at offset s % blockSize.  Only the blockNum dimension may  */
/* be non-contiguous ([EPI] 约束说明, [IDX] 约束说明), so a block is        */
/* blockSize rows of row_bytes bytes and blocks are block_stride apart.     */
/* ------------------------------------------------------------------------ */
typedef struct {
    uint8_t* base;
    int64_t num_blocks;
    int64_t block_size;
    int64_t row_bytes;
    int64_t block_stride;
} kvqo_paged;

static uint8_t* slot_row(const kvqo_paged* c, int64_t s)
{
    return c->base + (s / c->block_size) * c->block_stride + (s % c->block_size) * c->row_bytes;
}

static int64_t num_slots(const kvqo_paged* c) { return c->num_blocks * c->block_size; }

/* Element input types. */
#define KVQO_IN_BF16 0
#define KVQO_IN_F16 1
#define KVQO_IN_I32 2
#define KVQO_IN_F32 3

static float load_half(const uint16_t* p, int64_t i, int dtype)
{
    return dtype == KVQO_IN_F16 ? f16_to_f32(p[i]) : bf16_to_f32(p[i]);
}

static float max_abs(const float* v, int64_t n)
{
    float a = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float m = fabsf(v[i]);
        if (m > a) a = m;
    }
    return a;
}

/* ======================================================================== */
/* [EPI] kv_compress_epilog                                                 */
/* ======================================================================== */

/* Bytes written per row, [EPI] 约束说明 (headDim constraint):               */
/*   concatCol = (d-64) + 128 + ceil((d-64)/64) * scaleBytes   modes 0, 1   */
/*               (scaleBytes 2 in mode 0, 1 in mode 1)                       */
/*   concatCol = 64 + (d-64)/2 + ((d-64)/G) * 2                mode 2        */
/*   kvCacheCol = concatCol rounded up to 32 bytes in modes 0 and 2, as is   */
/*   in mode 1.  Worked example on the page: d=256, mode 1 -> 323.           */
int64_t kvqo_kv_cache_col(int64_t d, int quant_mode, int64_t group_size)
{
    int64_t n = d - 64;
    int64_t concat;
    if (quant_mode == 0 || quant_mode == 1) {
        int64_t scale_bytes = quant_mode == 0 ? 2 : 1;
        concat = n + 128 + ((n + 63) / 64) * scale_bytes;
    } else if (quant_mode == 2) {
        if (group_size <= 0) return -1;
        concat = 64 + n / 2 + (n / group_size) * 2;
    } else {
        return -1;
    }
    if (quant_mode == 1) return concat;
    return (concat + 31) / 32 * 32;
}

/*
 * One token row (d elements, bf16, or f16 in modes 0/1) -> packed cache row
 * of kvCacheCol bytes.
 *
 * Formula ([EPI] 计算公式):
 *   mode 0: groups of 64 over the nope columns [0, d-64):
 *           scale_g = max|x_g| / FP8_MAX,  q_i = round(x_i / scale_g);
 *           scale stored in 2 bytes (bfloat16), the rope columns kept bf16.
 *   mode 1: as mode 0 with the scale stored as E8M0, rounded up to a power
 *           of two.
 *   mode 2: rope (last 64 columns) static: rope_i = fp8(x_i * xScale);
 *           nope groups of G: scale_g = max|x_g| / FP4_MAX,
 *           nope_i = E2M1(x_i / scale_g), scales in 2 bytes.
 * Readings: round() is round-to-nearest-even to the target format with
 * saturation at its largest finite value; the division uses the STORED scale
 * (the bf16 value, or the exact power of two); a stored bf16 scale of zero
 * gives all-zero codes; hifloat8 (a format without an NVIDIA type) is
 * replaced by FP8 E4M3; the 2-byte scales are bfloat16.
 * Row layout (parity unpinned: a convention): [nope codes][rope][scales]
 * then zero bytes up to kvCacheCol.  FP4 codes two per byte, the even
 * element in the low nibble.  In modes 0/1 the rope columns are kept
 * unchanged: their 16-bit input values (bf16 or f16, `raw`) are copied,
 * little-endian; the 2-byte scale of mode 0 is bfloat16 whatever x's dtype
 * (the page names the mode "group (bf16 scale)").
 */
static void compress_row(const float* x, const uint16_t* raw, int64_t d, int quant_mode, int64_t G,
                         float x_scale, uint8_t* row, int64_t col)
{
    const int64_t n = d - 64;
    memset(row, 0, (size_t)col);
    if (quant_mode == 0 || quant_mode == 1) {
        const int64_t ngroups = n / 64;
        uint8_t* scales = row + n + 128;
        for (int64_t g = 0; g < ngroups; ++g) {
            const float* xg = x + 64 * g;
            float a = max_abs(xg, 64);
            if (quant_mode == 0) {
                float s = a / 448.0f;
                uint16_t sb = f32_to_bf16(s);
                float sf = bf16_to_f32(sb);
                scales[2 * g + 0] = (uint8_t)(sb & 0xFF);
                scales[2 * g + 1] = (uint8_t)(sb >> 8);
                for (int64_t i = 0; i < 64; ++i) {
                    row[64 * g + i] = (sf == 0.0f) ? 0u : enc_e4m3(xg[i] / sf);
                }
            } else {
                uint8_t b = e8m0_ceil(a / 448.0f);
                scales[g] = b;
                float mul = pow2f(127 - (int)b);   /* x / 2^(b-127), exact */
                for (int64_t i = 0; i < 64; ++i) row[64 * g + i] = enc_e4m3(xg[i] * mul);
            }
        }
        /* rope columns copied unchanged (the input's own 16-bit values), little-endian */
        for (int64_t j = 0; j < 64; ++j) {
            uint16_t h = raw[n + j];
            row[n + 2 * j + 0] = (uint8_t)(h & 0xFF);
            row[n + 2 * j + 1] = (uint8_t)(h >> 8);
        }
    } else {
        const int64_t ngroups = n / G;
        uint8_t* rope = row + n / 2;
        uint8_t* scales = row + n / 2 + 64;
        for (int64_t g = 0; g < ngroups; ++g) {
            const float* xg = x + G * g;
            float a = max_abs(xg, G);
            float s = a / 6.0f;
            uint16_t sb = f32_to_bf16(s);
            float sf = bf16_to_f32(sb);
            scales[2 * g + 0] = (uint8_t)(sb & 0xFF);
            scales[2 * g + 1] = (uint8_t)(sb >> 8);
            for (int64_t i = 0; i < G; ++i) {
                int64_t e = G * g + i;
                uint8_t c = (sf == 0.0f) ? 0u : enc_e2m1(xg[i] / sf);
                row[e / 2] |= (uint8_t)(c << (4 * (e % 2)));
            }
        }
        for (int64_t j = 0; j < 64; ++j) rope[j] = enc_e4m3(x[n + j] * x_scale);
    }
}

int kvqo_kv_compress_epilog(const uint16_t* x, int x_dtype, int64_t T, int64_t d, int64_t x_row_stride,
                            const int64_t* slot_mapping, const kvqo_paged* cache, int quant_mode,
                            int64_t quant_group_size, float x_scale, uint32_t* faults)
{
    if (d <= 64 || d % 64 != 0 || d > 8192) return KVQO_EINVAL;
    if (x_dtype != KVQO_IN_BF16 && x_dtype != KVQO_IN_F16) return KVQO_EINVAL;
    if (quant_mode == 2 && x_dtype != KVQO_IN_BF16) return KVQO_EINVAL;   /* mode 2 needs bf16 x */
    if (quant_mode == 2) {
        if (quant_group_size != 16 && quant_group_size != 32 && quant_group_size != 64) return KVQO_EINVAL;
        if ((d - 64) % quant_group_size != 0) return KVQO_EINVAL;
    }
    int64_t col = kvqo_kv_cache_col(d, quant_mode, quant_group_size);
    if (col < 0 || col > cache->row_bytes) return KVQO_EINVAL;
    float* xf = (float*)malloc(sizeof(float) * (size_t)d);
    uint8_t* row = (uint8_t*)malloc((size_t)col);
    if (!xf || !row) { free(xf); free(row); return KVQO_EINVAL; }
    for (int64_t t = 0; t < T; ++t) {
        int64_t s = slot_mapping[t];
        if (s == -1) continue;                               /* skipped token */
        if (s < 0 || s >= num_slots(cache)) { *faults |= KVQO_FAULT_SLOT_RANGE; continue; }
        for (int64_t i = 0; i < d; ++i) xf[i] = load_half(x + t * x_row_stride, i, x_dtype);
        compress_row(xf, x + t * x_row_stride, d, quant_mode, quant_group_size, x_scale, row, col);
        memcpy(slot_row(cache, s), row, (size_t)col);
    }
    free(xf);
    free(row);
    return KVQO_OK;
}

/* ------------------------------------------------------------------------ */
/* Packed-row decoder: the inverse of compress_row, as the attention side   */
/* reads the cache ([DRQ] 两种 KV Cache 更新模式: the cache rows are what    */
/* attention consumes).  Each code is decoded exactly (decode_bits), scaled */
/* by its group's stored scale with one binary32 multiply and rounded to    */
/* bf16 (round to nearest even):                                            */
/*   modes 0/1: nope y_i = bf16(fp8(q_i) * scale_g)  (scale_g: the bf16      */
/*              value, or 2^(b-127) for the E8M0 byte b); rope: the stored   */
/*              bf16 values;                                                 */
/*   mode 2:    nope y_i = bf16(e2m1(q_i) * scale_g); rope                   */
/*              y_j = bf16(fp8(r_j) / xScale), one IEEE division (the        */
/*              inverse of the static multiply).                             */
/* Readings: the pages define only the encoding; decoding with the stored   */
/* scale and one rounding to bf16 is the plain inverse.                     */
/* ------------------------------------------------------------------------ */
static uint16_t round_out(int y_dtype, float v) { return y_dtype == KVQO_IN_F16 ? f32_to_f16(v) : f32_to_bf16(v); }

static void decompress_row(const uint8_t* row, int64_t d, int quant_mode, int64_t G, float x_scale, int y_dtype,
                           uint16_t* y)
{
    const int64_t n = d - 64;
    if (quant_mode == 0 || quant_mode == 1) {
        const uint8_t* scales = row + n + 128;
        for (int64_t g = 0; g < n / 64; ++g) {
            float sf;
            if (quant_mode == 0) {
                uint16_t sb = (uint16_t)(scales[2 * g] | (scales[2 * g + 1] << 8));
                sf = bf16_to_f32(sb);
            } else {
                sf = (float)ldexp(1.0, (int)scales[g] - 127);   /* exact: 2^-127 .. 2^127 */
            }
            for (int64_t i = 0; i < 64; ++i) {
                float v = decode_bits(&FMT_E4M3, row[64 * g + i]);
                y[64 * g + i] = round_out(y_dtype, v * sf);
            }
        }
        for (int64_t j = 0; j < 64; ++j) y[n + j] = (uint16_t)(row[n + 2 * j] | (row[n + 2 * j + 1] << 8));
    } else {
        const uint8_t* rope = row + n / 2;
        const uint8_t* scales = row + n / 2 + 64;
        for (int64_t g = 0; g < n / G; ++g) {
            uint16_t sb = (uint16_t)(scales[2 * g] | (scales[2 * g + 1] << 8));
            float sf = bf16_to_f32(sb);
            for (int64_t i = 0; i < G; ++i) {
                int64_t e = G * g + i;
                uint32_t c = (row[e / 2] >> (4 * (e % 2))) & 0xFu;
                y[e] = f32_to_bf16(decode_bits(&FMT_E2M1, c) * sf);
            }
        }
        for (int64_t j = 0; j < 64; ++j) y[n + j] = f32_to_bf16(decode_bits(&FMT_E4M3, rope[j]) / x_scale);
    }
}

/* Decode the rows of slot_mapping into y [T, d] (row stride y_row_stride   */
/* elements; bf16, or f16 in modes 0/1 -- the dtype of the x that was       */
/* compressed, whose rope bytes the row holds).  Tokens whose slot is -1    */
/* leave their y row untouched; other slots outside the cache also leave it */
/* and raise the fault bit.                                                 */
int kvqo_kv_decompress(const kvqo_paged* cache, const int64_t* slot_mapping, int64_t T, int64_t d,
                       int quant_mode, int64_t quant_group_size, float x_scale, int y_dtype, uint16_t* y,
                       int64_t y_row_stride, uint32_t* faults)
{
    if (d <= 64 || d % 64 != 0 || d > 8192) return KVQO_EINVAL;
    if (y_dtype != KVQO_IN_BF16 && y_dtype != KVQO_IN_F16) return KVQO_EINVAL;
    if (quant_mode == 2 && y_dtype != KVQO_IN_BF16) return KVQO_EINVAL;
    if (quant_mode < 0 || quant_mode > 2) return KVQO_EINVAL;
    if (quant_mode == 2) {
        if (quant_group_size != 16 && quant_group_size != 32 && quant_group_size != 64) return KVQO_EINVAL;
        if ((d - 64) % quant_group_size != 0) return KVQO_EINVAL;
    }
    int64_t col = kvqo_kv_cache_col(d, quant_mode, quant_group_size);
    if (col < 0 || col > cache->row_bytes) return KVQO_EINVAL;
    for (int64_t t = 0; t < T; ++t) {
        int64_t s = slot_mapping[t];
        if (s == -1) continue;
        if (s < 0 || s >= num_slots(cache)) { *faults |= KVQO_FAULT_SLOT_RANGE; continue; }
        decompress_row(slot_row(cache, s), d, quant_mode, quant_group_size, x_scale, y_dtype, y + t * y_row_stride);
    }
    return KVQO_OK;
}

/* ======================================================================== */
/* [IDX] indexer_quant_cache                                                */
/* ======================================================================== */

/* quant_mode numbering: 0 mxfp8 (printed on the page), then 1 fp8,        */
/* 2 hifloat8, 3 mxfp4 in the order the page lists the modes (a reading).   */
#define KVQO_IDX_MXFP8 0
#define KVQO_IDX_FP8 1
#define KVQO_IDX_HIF8 2
#define KVQO_IDX_MXFP4 3

/* scaleCol: ceil(d/32) for the mx modes, 1 for fp8 / hifloat8.  Worked    */
/* example on the page: d=128, mode 0 -> 4.                                 */
int64_t kvqo_indexer_scale_col(int64_t d, int quant_mode)
{
    if (quant_mode == KVQO_IDX_MXFP8 || quant_mode == KVQO_IDX_MXFP4) return (d + 31) / 32;
    if (quant_mode == KVQO_IDX_FP8 || quant_mode == KVQO_IDX_HIF8) return 1;
    return -1;
}

/*
 * mxfp8 / mxfp4: groups of 32 elements, scale b = E8M0 rounded up of
 * max|x_g| / FP_MAX (FP8_MAX of the cache's FP8 format, 6 for FP4), codes
 * fp(x_i / 2^(b-127)); fp8: one group per row, scale = max|x| / FP8_MAX kept
 * as binary32, codes fp8(x_i / scale), all-zero codes when the scale is 0.
 * cache row: d code bytes (fp8) or ceil(d/2) bytes (fp4, even element in
 * the low nibble); cache_scale row: ceil(d/32) E8M0 bytes or one binary32.
 */
int kvqo_indexer_quant_cache(const uint16_t* x, int x_dtype, int64_t T, int64_t d, int64_t x_row_stride,
                             const int64_t* slot_mapping, const kvqo_paged* cache, int cache_fp8_fmt,
                             const kvqo_paged* cache_scale, int quant_mode, uint32_t* faults)
{
    if (d <= 0) return KVQO_EINVAL;
    if (quant_mode != KVQO_IDX_MXFP8 && quant_mode != KVQO_IDX_FP8 && quant_mode != KVQO_IDX_MXFP4)
        return KVQO_EINVAL;
    const kvqo_fmt* f8 = cache_fp8_fmt == 1 ? &FMT_E5M2 : &FMT_E4M3;
    const float fp8_max = (float)f8->maxval;
    const int64_t code_bytes = quant_mode == KVQO_IDX_MXFP4 ? (d + 1) / 2 : d;
    const int64_t scol = kvqo_indexer_scale_col(d, quant_mode);
    const int64_t scale_bytes = quant_mode == KVQO_IDX_FP8 ? 4 : scol;
    if (code_bytes > cache->row_bytes || scale_bytes > cache_scale->row_bytes) return KVQO_EINVAL;
    if (num_slots(cache) != num_slots(cache_scale)) return KVQO_EINVAL;
    float* xf = (float*)malloc(sizeof(float) * (size_t)d);
    uint8_t* codes = (uint8_t*)malloc((size_t)code_bytes);
    uint8_t* scales = (uint8_t*)malloc((size_t)scale_bytes);
    if (!xf || !codes || !scales) { free(xf); free(codes); free(scales); return KVQO_EINVAL; }
    for (int64_t t = 0; t < T; ++t) {
        int64_t s = slot_mapping[t];
        if (s == -1) continue;
        if (s < 0 || s >= num_slots(cache)) { *faults |= KVQO_FAULT_SLOT_RANGE; continue; }
        for (int64_t i = 0; i < d; ++i) xf[i] = load_half(x, t * x_row_stride + i, x_dtype);
        memset(codes, 0, (size_t)code_bytes);
        if (quant_mode == KVQO_IDX_FP8) {
            float a = max_abs(xf, d);
            float scale = a / fp8_max;
            for (int64_t i = 0; i < d; ++i)
                codes[i] = scale == 0.0f ? 0u : (uint8_t)encode_rn(f8, xf[i] / scale, 1);
            memcpy(scales, &scale, 4);
        } else {
            const float fmax = quant_mode == KVQO_IDX_MXFP8 ? fp8_max : 6.0f;
            for (int64_t g = 0; g < scol; ++g) {
                int64_t lo = 32 * g;
                int64_t len = (d - lo) < 32 ? (d - lo) : 32;
                float a = max_abs(xf + lo, len);
                uint8_t b = e8m0_ceil(a / fmax);
                scales[g] = b;
                float mul = pow2f(127 - (int)b);
                for (int64_t i = lo; i < lo + len; ++i) {
                    if (quant_mode == KVQO_IDX_MXFP8) {
                        codes[i] = (uint8_t)encode_rn(f8, xf[i] * mul, 1);
                    } else {
                        uint8_t c = enc_e2m1(xf[i] * mul);
                        codes[i / 2] |= (uint8_t)(c << (4 * (i % 2)));
                    }
                }
            }
        }
        memcpy(slot_row(cache, s), codes, (size_t)code_bytes);
        memcpy(slot_row(cache_scale, s), scales, (size_t)scale_bytes);
    }
    free(xf);
    free(codes);
    free(scales);
    return KVQO_OK;
}

/* ======================================================================== */
/* Static quantisation of one value into a cache element of a given dtype. */
/* ======================================================================== */
#define KVQO_C_BF16 0
#define KVQO_C_F16 1
#define KVQO_C_E4M3 2
#define KVQO_C_E5M2 3
#define KVQO_C_I8 4

/* Store y into element j of a cache row.  Unquantised caches take y      */
/* rounded to their dtype; quantised ones the static quantisation          */
/* q = fmt(y / scale) (+ offset before the int8 rounding), following the   */
/* Div -> Add offset -> Cast order of [DRQ] Kernel 实现要点.                 */
static void store_elem(uint8_t* row, int64_t j, int dt, float y, float scale, float offset, int has_offset)
{
    switch (dt) {
        case KVQO_C_BF16: {
            uint16_t h = f32_to_bf16(y);
            row[2 * j] = (uint8_t)(h & 0xFF);
            row[2 * j + 1] = (uint8_t)(h >> 8);
            break;
        }
        case KVQO_C_F16: {
            uint16_t h = f32_to_f16(y);
            row[2 * j] = (uint8_t)(h & 0xFF);
            row[2 * j + 1] = (uint8_t)(h >> 8);
            break;
        }
        case KVQO_C_E4M3: row[j] = enc_e4m3(y / scale); break;
        case KVQO_C_E5M2: row[j] = enc_e5m2(y / scale); break;
        case KVQO_C_I8: {
            float v = y / scale;
            if (has_offset) v = v + offset;
            row[j] = (uint8_t)int8_static(v);
            break;
        }
        default: break;
    }
}

/* ======================================================================== */
/* [RMS] kv_rmsnorm_rope_cache                                              */
/* ======================================================================== */

/* cache_mode values */
#define KVQO_RMS_NORM 0
#define KVQO_RMS_PA 1
#define KVQO_RMS_PA_BNSD 2
#define KVQO_RMS_PA_BLK_BNSD 3

typedef struct {
    kvqo_paged geom;
    int dtype;              /* KVQO_C_* */
    const float* scale;     /* NULL, 1 value (per tensor) or one per channel */
    int64_t scale_n;
    const float* offset;    /* NULL or like scale (int8 caches only) */
    int64_t offset_n;
} kvqo_cache_out;

static float param_at(const float* p, int64_t n, int64_t j) { return n == 1 ? p[0] : p[j]; }

/*
 * RMSNorm of the first Dv columns ([RMS] 计算公式 (2) rmsNorm):
 *   square_x = x*x; mean = mean(square_x); rms = sqrt(mean + eps);
 *   y = (x / rms) * gamma
 * Reading for the summation order, which the page leaves open: element i
 * belongs to 8-element chunk i/8; chunk c is owned by lane c mod 32; each
 * of 32 lanes sums its elements in increasing index order into a binary32
 * accumulator starting at 0; the 32 partial sums are then combined by the
 * butterfly p[l] = p[l] + p[l xor k] for k = 16, 8, 4, 2, 1; lane 0 holds the
 * sum.  For bf16 and f16 inputs x*x is exact in binary32.
 */
static void rmsnorm(const float* x, int64_t Dv, const float* gamma, float eps, float* y)
{
    float part[32];
    for (int l = 0; l < 32; ++l) part[l] = 0.0f;
    for (int64_t i = 0; i < Dv; ++i) {
        int l = (int)((i / 8) % 32);
        float sq = x[i] * x[i];
        part[l] = part[l] + sq;
    }
    for (int k = 16; k >= 1; k /= 2) {
        float nxt[32];
        for (int l = 0; l < 32; ++l) nxt[l] = part[l] + part[l ^ k];
        for (int l = 0; l < 32; ++l) part[l] = nxt[l];
    }
    float mean = part[0] / (float)Dv;
    float rms = sqrtf(mean + eps);
    for (int64_t i = 0; i < Dv; ++i) y[i] = (x[i] / rms) * gamma[i];
}

/*
 * Interleaved RoPE of the last Dk columns ([RMS] 计算公式 (1)):
 *   x1 = x[::2], x2 = x[1::2]; part1 = cat(x1, x2); part2 = cat(-x2, x1);
 *   y = part1 * cos + part2 * sin
 * so y_j = x_{2j} cos_j - x_{2j+1} sin_j and
 *    y_{h+j} = x_{2j+1} cos_{h+j} + x_{2j} sin_{h+j}, h = Dk/2.
 * The output is in the de-interleaved order the formula produces.
 */
static void rope_interleaved(const float* z, int64_t Dk, const float* c, const float* s, float* y)
{
    int64_t h = Dk / 2;
    for (int64_t j = 0; j < h; ++j) {
        float x1 = z[2 * j], x2 = z[2 * j + 1];
        y[j] = x1 * c[j] + (-x2) * s[j];
        y[h + j] = x2 * c[h + j] + x1 * s[h + j];
    }
}

static void write_cache_row(const kvqo_cache_out* co, int64_t slot, const float* y, int64_t n)
{
    uint8_t* row = slot_row(&co->geom, slot);
    for (int64_t j = 0; j < n; ++j) {
        float sc = co->scale ? param_at(co->scale, co->scale_n, j) : 1.0f;
        float of = co->offset ? param_at(co->offset, co->offset_n, j) : 0.0f;
        store_elem(row, j, co->dtype, y[j], sc, of, co->offset != NULL);
    }
}

/*
 * kv [B, 1, S, D] (N = 1), gamma [Dv], cos/sin [B, 1, S, Dk].  Index modes
 * ([RMS] 约束说明, index 相关约束):
 *   Norm:        index [B, S] in [-1, Scache); row = cache[b, 0, index].
 *                The caller passes the cache as blocks of Scache rows, one
 *                block per batch, so the slot is b * Scache + index.
 *   PA, PA_BNSD: index [B*S] in [-1, blockNum*blockSize); slot = index.
 *   PA_BLK_BNSD: index [B * ceil(S/blockSize)]; token (b, s) takes
 *                v = index[b*ceil(S/bs) + s/bs] and goes to block v/bs at
 *                offset s mod bs (reading: v names a block through v/bs).
 * -1 skips the token.  RMSNorm output -> ckv cache, RoPE output -> k cache.
 */
int kvqo_kv_rmsnorm_rope_cache(const uint16_t* kv, int kv_dtype, int64_t B, int64_t S, int64_t D, int64_t Dv,
                               const uint16_t* gamma, const uint16_t* cos, const uint16_t* sin,
                               const int64_t* index, int cache_mode, const kvqo_cache_out* k_out,
                               const kvqo_cache_out* ckv_out, float eps, uint32_t* faults)
{
    const int64_t Dk = D - Dv;
    if (Dv <= 0 || Dk <= 0 || Dk % 2 != 0) return KVQO_EINVAL;
    if (k_out->geom.block_size != ckv_out->geom.block_size || k_out->geom.num_blocks != ckv_out->geom.num_blocks)
        return KVQO_EINVAL;
    float* xf = (float*)malloc(sizeof(float) * (size_t)D);
    float* g = (float*)malloc(sizeof(float) * (size_t)Dv);
    float* cs = (float*)malloc(sizeof(float) * (size_t)Dk);
    float* sn = (float*)malloc(sizeof(float) * (size_t)Dk);
    float* yv = (float*)malloc(sizeof(float) * (size_t)Dv);
    float* yk = (float*)malloc(sizeof(float) * (size_t)Dk);
    if (!xf || !g || !cs || !sn || !yv || !yk) {
        free(xf); free(g); free(cs); free(sn); free(yv); free(yk);
        return KVQO_EINVAL;
    }
    for (int64_t i = 0; i < Dv; ++i) g[i] = load_half(gamma, i, kv_dtype);
    const int64_t bs = k_out->geom.block_size;
    const int64_t nslots = num_slots(&k_out->geom);
    const int64_t nblk_per_b = (S + bs - 1) / bs;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t si = 0; si < S; ++si) {
            const int64_t t = b * S + si;
            int64_t slot;
            if (cache_mode == KVQO_RMS_NORM) {
                int64_t v = index[t];
                if (v == -1) continue;
                if (v < 0 || v >= bs || b >= k_out->geom.num_blocks) { *faults |= KVQO_FAULT_SLOT_RANGE; continue; }
                slot = b * bs + v;
            } else if (cache_mode == KVQO_RMS_PA || cache_mode == KVQO_RMS_PA_BNSD) {
                slot = index[t];
                if (slot == -1) continue;
                if (slot < 0 || slot >= nslots) { *faults |= KVQO_FAULT_SLOT_RANGE; continue; }
            } else if (cache_mode == KVQO_RMS_PA_BLK_BNSD) {
                int64_t v = index[b * nblk_per_b + si / bs];
                if (v == -1) continue;
                if (v < 0 || v >= nslots) { *faults |= KVQO_FAULT_SLOT_RANGE; continue; }
                slot = (v / bs) * bs + si % bs;
            } else {
                free(xf); free(g); free(cs); free(sn); free(yv); free(yk);
                return KVQO_EINVAL;
            }
            for (int64_t i = 0; i < D; ++i) xf[i] = load_half(kv, t * D + i, kv_dtype);
            for (int64_t j = 0; j < Dk; ++j) {
                cs[j] = load_half(cos, t * Dk + j, kv_dtype);
                sn[j] = load_half(sin, t * Dk + j, kv_dtype);
            }
            rmsnorm(xf, Dv, g, eps, yv);
            rope_interleaved(xf + Dv, Dk, cs, sn, yk);
            write_cache_row(ckv_out, slot, yv, Dv);
            write_cache_row(k_out, slot, yk, Dk);
        }
    }
    free(xf); free(g); free(cs); free(sn); free(yv); free(yk);
    return KVQO_OK;
}

/* ======================================================================== */
/* [DRQ] dequant_rope_quant_kvcache                                         */
/* ======================================================================== */

typedef struct {
    /* x: [B, S, H] (S = 1 for a 2-D x), element type KVQO_IN_*            */
    const void* x;
    int x_dtype;
    int64_t B, S, H;
    /* cos / sin: [B, S, 1, D], element type bf16 or f16 (cos_dtype)       */
    const uint16_t* cos;
    const uint16_t* sin;
    int cos_dtype;
    /* caches: int8 [c0, c1, Nkv, D]; rows of Nkv*D bytes                   */
    uint8_t* k_cache;
    uint8_t* v_cache;
    int64_t c0, c1;
    int64_t k_block_stride, v_block_stride;   /* bytes between index-0 rows */
    const int64_t* indices;
    const float* scale_k;      /* [Nkv*D] */
    const float* scale_v;
    const float* offset_k;     /* optional */
    const float* offset_v;
    const float* weight_scale; /* [H], required for int32 x */
    const float* activation_scale; /* [B*S], optional */
    const void* bias;          /* [H], optional */
    int bias_dtype;            /* KVQO_IN_F32, KVQO_IN_F16, KVQO_IN_BF16, KVQO_IN_I32 */
    int64_t size_splits[3];    /* {Nq*D, Nkv*D, Nkv*D} */
    int64_t D;
    int cache_mode;            /* 0 contiguous, 1 page */
    int kv_output;
    uint16_t* q_out;           /* [B, S, Nq, D] in cos dtype */
    uint16_t* k_out;           /* [B, S, Nkv, D] when kv_output */
    uint16_t* v_out;
} kvqo_drq_args;

static float bias_at(const void* p, int dt, int64_t h)
{
    switch (dt) {
        case KVQO_IN_F32: return ((const float*)p)[h];
        case KVQO_IN_F16: return f16_to_f32(((const uint16_t*)p)[h]);
        case KVQO_IN_BF16: return bf16_to_f32(((const uint16_t*)p)[h]);
        case KVQO_IN_I32: return (float)((const int32_t*)p)[h];
        default: return 0.0f;
    }
}

static uint16_t round_to(int dt, float v) { return dt == KVQO_IN_F16 ? f32_to_f16(v) : f32_to_bf16(v); }

/*
 * Per token t = (b, s):
 *   1 dequant ([DRQ] 第 1 步, Kernel 实现要点 反量化): int32 x is cast to
 *     binary32, multiplied by weight_scale[h] (Mul), by activation_scale[t]
 *     (Muls, when given) and bias[h] is added (Add, when given), in that
 *     order.  A bf16 / f16 x is only widened.
 *   2 split ([DRQ] 第 2 步): q = [0, Nq*D), k = [Nq*D, (Nq+Nkv)*D), v = rest.
 *   3 RoPE ([DRQ] 第 3 步, Kernel 实现要点 RoPE): for each head u of q and k,
 *     h = D/2: o_j = u_j c_j + u_{j+h} (-s_j), o_{j+h} = u_{j+h} c_{j+h} + u_j s_{j+h}
 *     (sin negated first, then two Mul and one Add).
 *   4 quant ([DRQ] 第 4 步, Kernel 实现要点 量化): for channel c of k (after
 *     RoPE, still binary32) and v: int8(clamp(rint(w / scale_c + offset_c))).
 *   5 cache write ([DRQ] 两种 KV Cache 更新模式):
 *     page:       view(-1, Nkv, D)[indices[t]] = quantK[t]  (indices [B*S])
 *     contiguous: kCache[b][indices[b] + s] = quantK[b, s]   (indices [B])
 *   qOut = RoPE(q) rounded to the cos dtype; kOut = RoPE(k), vOut = v in the
 *   cos dtype when kv_output.
 * Readings: no intermediate rounding to 16 bits before the quantisation;
 * an index of -1 skips the token (as in the other three operations); other
 * out-of-range indices skip the token and raise the fault bit.
 */
int kvqo_dequant_rope_quant_kvcache(const kvqo_drq_args* a, uint32_t* faults)
{
    const int64_t D = a->D;
    if (D <= 0 || D % 2 != 0) return KVQO_EINVAL;
    const int64_t qw = a->size_splits[0], kw = a->size_splits[1], vw = a->size_splits[2];
    if (qw % D || kw % D || vw % D || kw != vw || qw + kw + vw != a->H) return KVQO_EINVAL;
    const int64_t Nq = qw / D, Nkv = kw / D, h = D / 2;
    const int64_t row_bytes = Nkv * D;
    const int64_t nslots = a->c0 * a->c1;
    float* w = (float*)malloc(sizeof(float) * (size_t)a->H);
    float* o = (float*)malloc(sizeof(float) * (size_t)a->H);
    float* cs = (float*)malloc(sizeof(float) * (size_t)D);
    float* sn = (float*)malloc(sizeof(float) * (size_t)D);
    if (!w || !o || !cs || !sn) { free(w); free(o); free(cs); free(sn); return KVQO_EINVAL; }
    for (int64_t b = 0; b < a->B; ++b) {
        for (int64_t s = 0; s < a->S; ++s) {
            const int64_t t = b * a->S + s;
            /* 1 dequant */
            for (int64_t i = 0; i < a->H; ++i) {
                const int64_t e = t * a->H + i;
                float v;
                if (a->x_dtype == KVQO_IN_I32) {
                    v = (float)((const int32_t*)a->x)[e];
                    v = v * a->weight_scale[i];
                    if (a->activation_scale) v = v * a->activation_scale[t];
                    if (a->bias) v = v + bias_at(a->bias, a->bias_dtype, i);
                } else {
                    v = load_half((const uint16_t*)a->x, e, a->x_dtype);
                }
                w[i] = v;
            }
            for (int64_t j = 0; j < D; ++j) {
                cs[j] = load_half(a->cos, t * D + j, a->cos_dtype);
                sn[j] = load_half(a->sin, t * D + j, a->cos_dtype);
            }
            /* 2 + 3: RoPE on the q and k heads; v passes through */
            for (int64_t hd = 0; hd < Nq + Nkv; ++hd) {
                const float* u = w + hd * D;
                float* out = o + hd * D;
                for (int64_t j = 0; j < h; ++j) {
                    float neg_s = -sn[j];
                    out[j] = u[j] * cs[j] + u[j + h] * neg_s;
                    out[j + h] = u[j + h] * cs[j + h] + u[j] * sn[j + h];
                }
            }
            for (int64_t i = qw + kw; i < a->H; ++i) o[i] = w[i];
            /* outputs in the cos dtype */
            for (int64_t i = 0; i < qw; ++i) a->q_out[t * qw + i] = round_to(a->cos_dtype, o[i]);
            if (a->kv_output) {
                for (int64_t i = 0; i < kw; ++i) a->k_out[t * kw + i] = round_to(a->cos_dtype, o[qw + i]);
                for (int64_t i = 0; i < vw; ++i) a->v_out[t * vw + i] = round_to(a->cos_dtype, o[qw + kw + i]);
            }
            /* 5: destination row */
            int64_t slot;
            if (a->cache_mode == 1) {
                slot = a->indices[t];
                if (slot == -1) continue;
                if (slot < 0 || slot >= nslots) { *faults |= KVQO_FAULT_SLOT_RANGE; continue; }
            } else {
                int64_t start = a->indices[b];
                if (start == -1) continue;
                int64_t pos = start + s;
                if (start < 0 || pos >= a->c1 || b >= a->c0) { *faults |= KVQO_FAULT_SLOT_RANGE; continue; }
                slot = b * a->c1 + pos;
            }
            uint8_t* krow = a->k_cache + (slot / a->c1) * a->k_block_stride + (slot % a->c1) * row_bytes;
            uint8_t* vrow = a->v_cache + (slot / a->c1) * a->v_block_stride + (slot % a->c1) * row_bytes;
            /* 4 quant */
            for (int64_t c = 0; c < kw; ++c) {
                float qk = o[qw + c] / a->scale_k[c];
                if (a->offset_k) qk = qk + a->offset_k[c];
                krow[c] = (uint8_t)int8_static(qk);
                float qv = o[qw + kw + c] / a->scale_v[c];
                if (a->offset_v) qv = qv + a->offset_v[c];
                vrow[c] = (uint8_t)int8_static(qv);
            }
        }
    }
    free(w); free(o); free(cs); free(sn);
    return KVQO_OK;
}
