/*
 * kvq.h -- C ABI of the B200 (sm_100a) per-token KV-cache epilogue library.
 *
 * One call per operation.  Each call validates its arguments on the host and,
 * if they are valid, enqueues exactly one kernel on the given CUDA stream and
 * returns.  Nothing is allocated, nothing is synchronised, no workspace is
 * needed; the caller owns every buffer.  Caches (and cache_scale) are updated
 * IN PLACE: only the rows addressed by a valid slot are written, and within a
 * row only the bytes the operation defines; every other byte keeps its value.
 * Execution is deterministic: each row has exactly one writer and no atomics
 * touch the outputs.
 *
 * Tensors are passed as kvq_tensor descriptors: a DEVICE pointer to element
 * [0, ..., 0], a dtype, and shape/stride in ELEMENTS (not bytes).  The
 * library never dereferences a descriptor's data on the host.
 *
 * Errors.  A host-detected problem (null pointer, wrong rank, shape, dtype,
 * attribute, layout or capacity) returns a nonzero kvq_status and launches
 * nothing.  After a launch the call returns KVQ_ERR_CUDA if that launch itself
 * failed (the status of the launch call; errors left by unrelated earlier CUDA
 * work are neither reported nor cleared), else KVQ_OK.  Data faults the
 * device can see -- a slot index outside [0, num_slots) that is not -1 --
 * skip the affected row and set a bit in a per-device fault word; a call's
 * KVQ_OK does not say that no such fault happened: callers that need to know
 * call kvq_get_error(), which returns and clears the bits.  Duplicate slots
 * are not detected (the pages declare the result undefined); rows then have
 * two writers and either may win.
 *
 * Sources (page title and section):
 *   aclnnKvCompressEpilog        -- 接口功能, 计算公式, 约束说明
 *   aclnnKvRmsNormRopeCache      -- 接口功能, 计算公式, 约束说明
 *   indexer_quant_cache          -- 接口功能, 语义说明, 约束说明 (torch_npu op)
 *   aclnnDequantRopeQuantKvcache 算子深度解析 -- 计算步骤公式, 两段式接口与函数原型,
 *                                   约束说明, Shape 推导逻辑, Kernel 实现要点
 * The pages' two-stage GetWorkspaceSize + execute pattern becomes one call:
 * the workspace is always 0 bytes and validation happens before the launch.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols of the ABI are exported; everything else in the library is hidden. */
#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

/* A CUDA stream (the same object as cudaStream_t / CUstream).  NULL is the
 * legacy default stream. */
struct CUstream_st;
typedef struct CUstream_st* kvq_stream;

typedef enum {
    KVQ_BF16 = 0,
    KVQ_F16 = 1,
    KVQ_F32 = 2,
    KVQ_I32 = 3,
    KVQ_I64 = 4,
    KVQ_I8 = 5,
    KVQ_U8 = 6,
    KVQ_F8E4M3 = 7,   /* FLOAT8 E4M3FN: no infinities, max 448 */
    KVQ_F8E5M2 = 8,   /* FLOAT8 E5M2: max finite 57344 */
    KVQ_E8M0 = 9      /* unsigned 8-bit power-of-two scale 2^(b-127) */
} kvq_dtype;

#define KVQ_MAX_DIMS 8

typedef struct {
    void* data;                       /* device pointer to element [0,...,0] */
    int32_t dtype;                    /* kvq_dtype */
    int32_t ndim;                     /* 0 .. KVQ_MAX_DIMS */
    int64_t shape[KVQ_MAX_DIMS];
    int64_t stride[KVQ_MAX_DIMS];     /* in elements */
} kvq_tensor;

typedef enum {
    KVQ_OK = 0,
    KVQ_ERR_NULL = 1,         /* a required tensor or its data pointer is NULL */
    KVQ_ERR_NDIM = 2,         /* wrong number of dimensions */
    KVQ_ERR_SHAPE = 3,        /* inconsistent sizes */
    KVQ_ERR_DTYPE = 4,        /* dtype not allowed here */
    KVQ_ERR_ATTR = 5,         /* bad attribute value (mode, group size, ...) */
    KVQ_ERR_LAYOUT = 6,       /* non-contiguous where contiguity is required */
    KVQ_ERR_CAPACITY = 7,     /* cache row (headDim) too small for the packed row */
    KVQ_ERR_CUDA = 8,         /* the CUDA runtime reported an error */
    KVQ_ERR_UNSUPPORTED = 9   /* a valid combination this library does not implement */
} kvq_status;

/* Fault bits of the device fault word. */
#define KVQ_FAULT_SLOT_RANGE 0x1u   /* a slot/index outside [0, num_slots) and not -1 */
#define KVQ_FAULT_TIMEOUT 0x2u      /* a pipeline wait gave up (an internal error; the output is incomplete) */

/* ------------------------------------------------------------------------ */
/* kv_compress_epilog                                                        */
/* Source: aclnnKvCompressEpilog, 接口功能 / 计算公式 / 约束说明.               */
/*                                                                           */
/* x            bf16 [..., d] (f16 also in quant_mode 0/1: the page requires  */
/*              bf16 only in mode 2); the last dimension contiguous, the      */
/*              leading dimensions flattenable to T rows with one row stride. */
/*              64 < d <= 8192, d % 64 == 0.  Columns [0, d-64) are the nope  */
/*              segment, [d-64, d) the rope segment.                          */
/* slot_mapping int32 or int64, T elements (x's leading dims flattened),     */
/*              contiguous.  -1 skips the token; other values in             */
/*              [0, blockNum*blockSize) and distinct.                         */
/* cache        uint8 [blockNum, blockSize, 1, headDim], headDim >= kvCacheCol */
/*              (kvq_kv_cache_col).  Rows contiguous inside a block; only    */
/*              the blockNum dimension may be strided.                        */
/* quant_mode   0: groups of 64 -> FP8 E4M3, bf16 scale = amax/448;          */
/*              1: groups of 64 -> FP8 E4M3, E8M0 scale = amax/448 rounded up */
/*                 to a power of two;                                         */
/*              2: nope groups of quant_group_size -> FP4 E2M1, bf16 scale =  */
/*                 amax/6; rope -> FP8 E4M3 of x * x_scale (this library's   */
/*                 stand-in for the pages' hifloat8).                         */
/* quant_group_size  16, 32 or 64 in mode 2 ((d-64) % G == 0); ignored else. */
/* x_scale      mode 2 rope multiplier; ignored else.                         */
/* Codes are round-to-nearest-even with saturation of x divided by the       */
/* STORED scale; a stored bf16 scale of 0 gives all-zero codes.              */
/* Packed row (kvCacheCol bytes, written from byte 0 of the slot row):       */
/*   modes 0/1: [d-64 code bytes][the 64 rope values as given: bf16 or f16   */
/*              bytes][(d-64)/64 scales: bf16 (mode 0, whatever x's dtype)   */
/*              or E8M0 (mode 1)]                                            */
/*   mode 2:    [(d-64)/2 bytes of FP4 pairs, even element in the low nibble] */
/*              [64 E4M3 rope codes][(d-64)/G bf16 scales]                   */
/*   then 0x00 up to kvCacheCol (32-byte alignment in modes 0 and 2).        */
/* ------------------------------------------------------------------------ */
KVQ_API kvq_status kvq_kv_compress_epilog(const kvq_tensor* x, const kvq_tensor* slot_mapping, kvq_tensor* cache,
                                  int32_t quant_mode, int32_t quant_group_size, float x_scale,
                                  kvq_stream stream);

/* ------------------------------------------------------------------------ */
/* kv_decompress: the packed-row decoder, the inverse of kv_compress_epilog  */
/* as the attention side reads the cache.  Source: the row layout and the    */
/* formulas of aclnnKvCompressEpilog (计算公式, 约束说明), read backwards;   */
/* the pages define only the encoding, so the decode is their plain inverse. */
/*                                                                           */
/* cache        uint8 [blockNum, blockSize, 1, headDim] written by            */
/*              kv_compress_epilog with the same quant_mode,                  */
/*              quant_group_size and x_scale (headDim >= kvCacheCol).         */
/* slot_mapping int32 or int64, T elements, contiguous: the slot of each     */
/*              output row; -1 leaves the row untouched.                      */
/* y            bf16 [..., d] (the last dimension contiguous, the leading     */
/*              dimensions flattenable to T rows with one row stride),        */
/*              written row by row; in modes 0/1 y may be f16 instead, for    */
/*              rows compressed from f16 x (y's dtype must be x's: the rope   */
/*              is stored as x's own 16-bit values):                          */
/*   modes 0/1: nope y = round_to_y(code value * group scale) (the bf16      */
/*              scale, or 2^(b-127) for the E8M0 byte b); rope = the stored  */
/*              16-bit values;                                                */
/*   mode 2:    nope y = bf16_rn(E2M1 value * group scale); rope =           */
/*              bf16_rn(E4M3 value / x_scale) (IEEE division).                */
/* Validation as kv_compress_epilog; a slot outside the cache leaves its row */
/* untouched and sets KVQ_FAULT_SLOT_RANGE (kvq_get_error).  The caller owns */
/* y; the call allocates nothing and enqueues one kernel on `stream`.        */
/* ------------------------------------------------------------------------ */
KVQ_API kvq_status kvq_kv_decompress(const kvq_tensor* cache, const kvq_tensor* slot_mapping, kvq_tensor* y,
                                     int32_t quant_mode, int32_t quant_group_size, float x_scale,
                                     kvq_stream stream);

/* Bytes of one packed row (kvCacheCol) for kv_compress_epilog, or -1 for an
 * invalid (d, quant_mode, quant_group_size).  Closed form of
 * aclnnKvCompressEpilog 约束说明 (headDim constraint); d=256, mode 1 -> 323. */
KVQ_API int64_t kvq_kv_cache_col(int64_t d, int32_t quant_mode, int32_t quant_group_size);

/* ------------------------------------------------------------------------ */
/* indexer_quant_cache                                                       */
/* Source: indexer_quant_cache, 接口功能 / 语义说明 / 约束说明.                 */
/*                                                                           */
/* x            bf16 or f16 [..., d], last dimension contiguous, leading dims */
/*              flattenable to T rows; 1 <= d <= 2^24 (else KVQ_ERR_SHAPE).   */
/* cache        [blockNum, blockSize, 1, headDim]: FLOAT8 E4M3 or E5M2 for    */
/*              mxfp8/fp8 (headDim >= d), uint8 for mxfp4 (headDim >=         */
/*              ceil(d/2) bytes, two E2M1 codes per byte, even element low).  */
/* cache_scale  [blockNum, blockSize, 1, scaleHeadDim] with the same blockNum */
/*              and blockSize: E8M0 (or uint8) for mxfp8/mxfp4, scaleHeadDim  */
/*              >= ceil(d/32); FLOAT32 for fp8, scaleHeadDim >= 1.            */
/* slot_mapping int32/int64, T elements, -1 skips.                            */
/* quant_mode   0 mxfp8 (groups of 32, E8M0 scale rounded up, codes          */
/*                FP8(x / 2^(b-127)), format from cache dtype);               */
/*              1 fp8 (one group per row, fp32 scale = amax / FP8_MAX);      */
/*              2 hifloat8 -> KVQ_ERR_UNSUPPORTED (no NVIDIA type);          */
/*              3 mxfp4 (groups of 32, E8M0 scale, E2M1 codes).               */
/* ------------------------------------------------------------------------ */
KVQ_API kvq_status kvq_indexer_quant_cache(const kvq_tensor* x, kvq_tensor* cache, kvq_tensor* cache_scale,
                                   const kvq_tensor* slot_mapping, int32_t quant_mode, kvq_stream stream);

/* scaleCol of indexer_quant_cache: ceil(d/32) for mxfp8/mxfp4, 1 for fp8 and
 * hifloat8, -1 otherwise.  The page's example: d=128, mode 0 -> 4. */
KVQ_API int64_t kvq_indexer_scale_col(int64_t d, int32_t quant_mode);

/* ------------------------------------------------------------------------ */
/* kv_rmsnorm_rope_cache                                                     */
/* Source: aclnnKvRmsNormRopeCache, 接口功能 / 计算公式 / 约束说明.             */
/*                                                                           */
/* kv        bf16 or f16 [B, 1, S, D] contiguous (N = 1).  D = Dv + Dk with   */
/*           Dv = ckv_cache's last dim, Dk = k_cache's last dim, Dk even,    */
/*           D <= 2^24 (else KVQ_ERR_SHAPE).                                   */
/* gamma     [Dv], same dtype as kv.                                          */
/* cos, sin  [B, 1, S, Dk], same dtype as kv, contiguous.                     */
/* index     int32/int64.  cache_mode 0 Norm: [B, S], values in [-1, Scache), */
/*           caches [Bc, 1, Scache, Dc] with Bc >= B; 1 PA and 2 PA_BNSD:     */
/*           [B*S], values in [-1, blockNum*blockSize), caches               */
/*           [blockNum, blockSize, 1, Dc] or [blockNum, 1, blockSize, Dc];   */
/*           3 PA_BLK_BNSD: [B*ceil(S/blockSize)], entry v places token s of  */
/*           batch b in block v/blockSize at offset s % blockSize.  -1 skips. */
/* k_cache   receives RoPE(kv[..., Dv:]) (interleaved pairs, de-interleaved   */
/* ckv_cache output order); ckv_cache receives RMSNorm(kv[..., :Dv]) * gamma. */
/*           dtypes: bf16/f16 (stored rounded to nearest even), or FLOAT8     */
/*           E4M3/E5M2 or int8 (static quantisation fp(y / scale), int8 also  */
/*           + offset, round half even, saturating); a quantised cache needs  */
/*           its scale tensor (f32, 1 or Dc elements); offsets only for int8. */
/*           blockSize % 32 == 0 for 1-byte caches, % 16 for 2-byte caches.   */
/* RMSNorm: rms = sqrt(mean(x*x) + epsilon), y = (x / rms) * gamma.  The sum */
/* of squares uses a fixed order: element i belongs to 8-element chunk i/8,   */
/* chunk c to lane c % 32; lanes add their elements in index order; the 32    */
/* partial sums combine by the butterfly p[l] += p[l ^ k], k = 16..1.         */
/* ------------------------------------------------------------------------ */
KVQ_API kvq_status kvq_kv_rmsnorm_rope_cache(const kvq_tensor* kv, const kvq_tensor* gamma, const kvq_tensor* cos,
                                     const kvq_tensor* sin, const kvq_tensor* index, kvq_tensor* k_cache,
                                     kvq_tensor* ckv_cache, const kvq_tensor* k_scale,
                                     const kvq_tensor* ckv_scale, const kvq_tensor* k_offset,
                                     const kvq_tensor* ckv_offset, float epsilon, int32_t cache_mode,
                                     kvq_stream stream);

/* ------------------------------------------------------------------------ */
/* dequant_rope_quant_kvcache                                                */
/* Source: aclnnDequantRopeQuantKvcache 算子深度解析, 计算步骤公式, 两种 KV     */
/* Cache 更新模式, 两段式接口与函数原型 (argument order), 约束说明, Shape 推导.   */
/*                                                                           */
/* x          int32, bf16 or f16, [B, S, H] or [B, H] (S = 1), contiguous.    */
/* cos, sin   bf16 or f16 [B, S, 1, D] (or [B, 1, D] / [B, 1, 1, D] for 2-D  */
/*            x), contiguous; for a 16-bit x the same dtype as x.            */
/* k_cache,   int8 [c0, c1, Nkv, D], (Nkv, D) contiguous, only dim 0 strided. */
/* v_cache    D % 32 == 0.                                                    */
/* indices    int32/int64.  page (cache_mode 1): [B*S], row                   */
/*            cache.view(-1, Nkv, D)[indices[t]], values in [0, c0*c1);       */
/*            contiguous (0): [B], token s of batch b -> cache[b][indices[b]+s]. */
/*            -1 skips (page mode: the token; contiguous: the batch).         */
/* scale_k, scale_v     f32, Nkv*D elements; offset_k/v optional, f32.        */
/* weight_scale         f32 [H], required for int32 x;                        */
/* activation_scale     f32 [B*S], optional; bias [H] optional, f32/f16/bf16/ */
/*                      int32.  For a 16-bit x these three are ignored.       */
/* size_splits          {Nq*D, Nkv*D, Nkv*D}, n_splits == 3, sum == H.        */
/* quant_mode 0 ("static"), layout 0 ("BSND") are the only values.            */
/* kv_output  nonzero: k_out / v_out [B, S, Nkv, D] (cos dtype) are written.  */
/* q_out      [B, S, Nq, D] (or [B, Nq, D]) in the cos dtype.                 */
/* Per token: v = ((float)x * weight_scale[h]) * activation_scale[t] + bias[h]; */
/* split; half-rotation RoPE on q and k heads: o_j = u_j c_j - u_{j+D/2} s_j,  */
/* o_{j+D/2} = u_{j+D/2} c_{j+D/2} + u_j s_{j+D/2}; int8 quantisation of k     */
/* (after RoPE, binary32) and v: clamp(rint(w / scale + offset), -128, 127).  */
/* ------------------------------------------------------------------------ */
KVQ_API kvq_status kvq_dequant_rope_quant_kvcache(const kvq_tensor* x, const kvq_tensor* cos, const kvq_tensor* sin,
                                          kvq_tensor* k_cache, kvq_tensor* v_cache, const kvq_tensor* indices,
                                          const kvq_tensor* scale_k, const kvq_tensor* scale_v,
                                          const kvq_tensor* offset_k, const kvq_tensor* offset_v,
                                          const kvq_tensor* weight_scale, const kvq_tensor* activation_scale,
                                          const kvq_tensor* bias, const int64_t* size_splits, int32_t n_splits,
                                          int32_t quant_mode, int32_t layout, int32_t kv_output,
                                          int32_t cache_mode, kvq_tensor* q_out, kvq_tensor* k_out,
                                          kvq_tensor* v_out, kvq_stream stream);

/* ------------------------------------------------------------------------ */
/* compressor: the token Compressor, C128A form (coff = 1) and C4A / C4Li   */
/* form (coff = 2, cmp_ratio = 4)                                            */
/* Source: aclnnCompressor, 接口功能 / 计算公式 steps 1-5 / 约束说明.          */
/*                                                                           */
/* C128A (w_kv [D, H]): per group i of cmp_ratio consecutive token rows and  */
/* per channel c:                                                            */
/*   kv_state = X @ W^KV^T, score_state = X @ W^Gate^T (step 1),             */
/*   s_r = score_state[r, c] + ape[r mod cmp_ratio, c] (step 2),             */
/*   p = softmax over the group's rows of s (step 3, channel by channel),    */
/*   cmp_kv[i, c] = sum_r p_r kv_state[r, c] (steps 4-5), rounded to bf16.   */
/* C4A (w_kv [2D, H], cmp_ratio 4): rows [0, D) of w_kv / w_gate are the a   */
/*   weights, rows [D, 2D) the b weights; group i takes its own four tokens  */
/*   4i .. 4i+3 through the a weights (scores + ape[p, c]) and the next four */
/*   4i+4 .. 4i+7 through the b weights (scores + ape[p, D + c]); the        */
/*   softmax and the sum run over those eight rows, and over the own four    */
/*   alone for the last group of the chunk (no next tokens).                 */
/* x       bf16 [..., H], contiguous, 16-byte aligned; the leading dims are   */
/*         the T token rows, T % cmp_ratio == 0 (whole groups: the stateless  */
/*         case; the page's state cache, start_pos and cu_seqlens are not     */
/*         modelled).  1024 <= H <= 10240, H % 512 == 0.                     */
/* w_kv,   bf16 [coff*D, H], contiguous, 16-byte aligned; D = 128 or 512;     */
/* w_gate  coff (1 or 2) follows from w_kv's rows and cmp_kv's D.             */
/* ape     f32 [cmp_ratio, coff*D], contiguous.                               */
/* cmp_kv  bf16 [T / cmp_ratio, D], contiguous: written.                     */
/* cmp_ratio  2, 4, 8, 16, 32, 64 or 128 (C128A: 128); 4 when coff = 2,       */
/*         else KVQ_ERR_ATTR.                                                 */
/* Arithmetic: bf16 products with fp32 accumulation on the tensor cores       */
/* (tcgen05), the softmax in fp32; the result is within the bound of fp32     */
/* accumulation of the exact value, not bit-reproducible against another      */
/* summation order.  One kernel on `stream`; nothing is allocated; no         */
/* workspace.  KVQ_ERR_CUDA if the TMA descriptors cannot be encoded.         */
/* ------------------------------------------------------------------------ */
KVQ_API kvq_status kvq_compressor(const kvq_tensor* x, const kvq_tensor* w_kv, const kvq_tensor* w_gate,
                                  const kvq_tensor* ape, kvq_tensor* cmp_kv, int32_t cmp_ratio, kvq_stream stream);

/* ------------------------------------------------------------------------ */
/* Utilities                                                                 */
/* ------------------------------------------------------------------------ */

/* Read and clear the current device's fault word: enqueues on `stream` one
 * kernel that atomically exchanges the word with 0 (after every earlier
 * kernel of the stream has completed), copies that value back, waits for
 * `stream` and stores the bits in *fault_bits.  Because the read and the
 * clear are one atomic operation, a bit raised by a kernel on another stream
 * is returned either by this call or by the next one, never lost.  Returns
 * KVQ_ERR_CUDA if the launch, the copy or the stream reported an error (the
 * bits are then 0). */
KVQ_API kvq_status kvq_get_error(kvq_stream stream, uint32_t* fault_bits);

/* Element-wise conversion of n binary32 values on the device with the same
 * device codecs the kernels use (no counterpart on the pages; it lets the
 * codecs be checked exhaustively).  fmt: 0 E4M3 (satfinite, 1 byte each),
 * 1 E5M2 (satfinite), 2 E2M1 (satfinite, one code per byte in the low
 * nibble), 3 bf16 (2 bytes, RNE), 4 E8M0 rounded up (1 byte), 5 int8 static
 * (1 byte, rint then clamp).  in, out: device pointers. */
KVQ_API kvq_status kvq_convert(int32_t fmt, const float* in, int64_t n, void* out, kvq_stream stream);

/* Device self-test of the arithmetic shortcuts the kernels rely on (no
 * counterpart on the pages).  which = 0 / 1: the number of (numerator, scale)
 * pairs -- every finite bf16 numerator a and every bf16 scale s in
 * [2^-100, 2^101) with |a| <= 512 s -- where the one-step (0) or two-step (1)
 * division-by-scale differs from IEEE division in any bit; 2 / 3: the number
 * of such pairs whose E4M3 (2) or E2M1 (3) code of the one-step quotient
 * differs from the code of the IEEE quotient; 4: the number of positive
 * finite bf16 and f16 values a for which the constant-divisor form of a / 448,
 * a / 57344 or a / 6 differs from IEEE division; 5: as 0 but counting only
 * pairs whose IEEE quotient is a normal binary32 number; 6: the number of
 * groups of four, among 2^28 random (value, scale, offset) triples (half of
 * them within a few ulps of a rounding tie), whose static int8 codes from the
 * dequant kernel's reciprocal-based quotient differ from those of IEEE
 * division; 7: the bounded wait of the pipelined kernels, run out on purpose
 * (a shared-memory barrier that nothing completes, a short limit): 1 when the
 * wait gave up as designed -- it also sets KVQ_FAULT_TIMEOUT, which
 * kvq_get_error returns and clears; 8: the number of (value, row maximum,
 * format) cases, among 2^28 random bf16 / f16 pairs with |value| <= maximum,
 * each encoded as E4M3 and as E5M2, whose code from the indexer fp8 mode's
 * two-step quotient by maximum / FP8_MAX differs from the code of the IEEE
 * quotient; 9: the number of (x, rms) pairs, among 2^28 random ones inside
 * the rmsnorm kernel's guard (rms in [2^-60, 2^50], x a bf16 value with |x| >=
 * max(RN(rms 2^-125), 2^-103), half of them within a few ulps of a rounding
 * tie), whose one-step quotient x / rms (q0 = RN(x r), r = RN(1/rms), then
 * RN(q0 + (x - q0 rms) r)) differs in any bit from IEEE division; 10: the
 * number of (numerator, divisor) pairs, every bf16 and every f16 numerator
 * mantissa of either sign against every binary32 divisor mantissa (both in
 * [1, 2)), whose one-step quotient differs in any bit from IEEE division.
 * Blocks until done; *result receives the count (0 means the shortcut is
 * exact on the domain). */
KVQ_API kvq_status kvq_selftest(int32_t which, uint64_t* result, kvq_stream stream);

/* The memory access pattern of kv_compress_epilog without its arithmetic (no
 * counterpart on the pages; a measuring stick for the compress kernels): for
 * each token t with slot s = slot_mapping[t] != -1, read the whole row t of x
 * (any dtype, [..., d] with the last dimension contiguous, d * element size a
 * multiple of 16 and at most 2048 bytes, rows 16-byte aligned) and write its
 * first out_bytes bytes (a multiple of 16, at most the row size) to the start
 * of slot row s of cache (uint8 [blockNum, blockSize, 1, headDim], headDim >=
 * out_bytes, rows 16-byte aligned; otherwise KVQ_ERR_LAYOUT).  Slots outside
 * the cache skip the row and set KVQ_FAULT_SLOT_RANGE.  One kernel on `stream`;
 * nothing is allocated. */
KVQ_API kvq_status kvq_scatter_rows(const kvq_tensor* x, const kvq_tensor* slot_mapping, kvq_tensor* cache,
                                    int64_t out_bytes, kvq_stream stream);

/* Static description of a status code. */
KVQ_API const char* kvq_status_string(kvq_status status);

/* Library version, major*10000 + minor*100 + patch. */
KVQ_API int32_t kvq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
