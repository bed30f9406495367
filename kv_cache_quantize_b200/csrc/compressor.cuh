// compressor.cuh -- the token Compressor (aclnnCompressor, 计算公式 steps 1-5,
// C128A form: coff = 1, groups of cmp_ratio consecutive tokens) as one
// tcgen05 kernel: the two projections on the tensor cores, the grouped
// softmax, the Hadamard product and the group sum in the epilogue.
//
// The product is computed transposed, D^T = W X^T: the UMMA M dimension is
// 128 channels (rows of W^KV and W^Gate), N is BN = 256 tokens (128 when the
// batch is small, for twice the tiles), K the hidden size.
// In tensor memory an accumulator row is then one channel and a column one
// token, so the softmax over the rows of a token group (step 3) runs along a
// single thread's TMEM row: no cross-thread reduction, and the scores never
// leave the SM.  Two accumulators share every X tile: kv_state in TMEM
// columns [0, BN), score_state in [BN, 2 BN) (all 512 columns of the SM at
// BN = 256).
//
// Roles (192 threads, one CTA per SM, persistent over tiles of 128 channels
// x BN tokens; the four channel tiles of a token tile are adjacent tile
// numbers, so they run together and read the X tile from L2 once):
//   warp 0, one lane: TMA producer -- a ring (3 stages at BN = 256, 4 at 128)
//     of K slices of 64 (W^KV 128x64, W^Gate 128x64 and X BNx64 bf16 boxes,
//     128-byte swizzle),
//     completion counted in bytes on the stage's `full` mbarrier;
//   warp 1: allocates TMEM; one lane issues tcgen05.mma (kind::f16, bf16 in,
//     fp32 accumulate, M 128, N BN, K 16) and commits each stage to its
//     `empty` barrier and each finished tile to `tmem_full`;
//   warps 2-5: the epilogue -- warp w reads TMEM lanes 32 (w % 4) .. +31 (the
//     lane quarter its hardware subpartition may access), i.e. 32 channels,
//     32 tokens per tcgen05.ld, and keeps per channel a running maximum, sum
//     of weights and weighted kv sum (online softmax), emitting one bf16
//     output per channel and group; then it frees the accumulators on
//     `tmem_empty`.
// No cluster, no multicast: every TMA load reads this GPU's own memory into
// this CTA.  Every wait is bounded (FAULT_TIMEOUT), and the MMA thread drains
// its tensor-core work before TMEM is released.
#pragma once

#include <cuda.h>

#include "kvq_device.cuh"
#include "tma_pipe.cuh"

namespace kvq {

constexpr int CP_BM = 128;                      // channels per tile (UMMA M)
constexpr int CP_BN = 256;                      // tokens per tile (UMMA N), the large-batch width
constexpr int CP_BK = 64;                       // K per stage: one 128-byte swizzle row of bf16
constexpr int CP_UK = 16;                       // K of one tcgen05.mma kind::f16
constexpr int CP_THREADS = 192;
constexpr uint32_t CP_A_BYTES = CP_BM * CP_BK * 2;                  // 16 KB

// the ring and tensor-memory shape for a token-tile width BN (256 or 128)
__host__ __device__ constexpr int cp_stages(int bn) { return bn == 256 ? 3 : 4; }
__host__ __device__ constexpr uint32_t cp_stage_bytes(int bn) { return 2 * CP_A_BYTES + (uint32_t)bn * CP_BK * 2; }
__host__ __device__ constexpr uint32_t cp_smem_bytes(int bn) {
    return (uint32_t)cp_stages(bn) * cp_stage_bytes(bn) + 256 + 1024;   // + barriers + alignment slack
}
constexpr uint64_t CP_WAIT_NS = 2000000000ull;     // every wait gives up after 2 s (a tile takes < 1 ms)

struct CompressorArgs {
    int64_t T;             // token rows (a multiple of ratio)
    int32_t H;             // hidden size (a multiple of 64)
    int32_t D;             // channels (a multiple of 128)
    int32_t n_ch_tiles;    // D / 128
    int64_t n_tok_tiles;   // ceil(T / BN)
    const float* ape;      // [ratio, D]
    uint16_t* out;         // bf16 [T / ratio, D]
};

// ---------------------------------------------------------------------------
// tcgen05 / TMA wrappers
// ---------------------------------------------------------------------------
// 2-D tiled TMA load of box {x (inner, elements), y} into this CTA's shared memory
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int32_t x, int32_t y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// 4-D tiled TMA load of box {x, y, z, w} (x innermost) into this CTA's shared memory
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int32_t x, int32_t y, int32_t z,
                                            int32_t w, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major bf16, fp32 accumulate
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// the mbarrier receives one arrival once every tcgen05 operation this thread
// issued before has completed
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Shared-memory matrix descriptor of a K-major bf16 tile written by TMA with
// the 128-byte swizzle: rows of 64 values (128 bytes) at a 128-byte pitch,
// groups of 8 rows 1024 bytes apart (stride byte offset), leading byte
// offset unused for this layout (1), descriptor version 1, layout type 2
// (128-byte swizzle).  The K slice k of a stage starts 32 k bytes in; the
// tile itself starts on a 1024-byte boundary.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits 4-5 = 1), A and B
// bf16 (bits 7-9 = 1, 10-12 = 1), both K-major (bits 15, 16 = 0), N / 8 in
// bits 17-22, M / 16 in bits 24-28.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// 32 consecutive fp32 columns at each of two TMEM addresses of this thread's
// lane, and the wait for both loads, in ONE asm statement: the outputs exist
// only after tcgen05.wait::ld, so no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_ld32x2(uint32_t ta, uint32_t tb, uint32_t (&ra)[32], uint32_t (&rb)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%65];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(ra[0]), "=r"(ra[1]), "=r"(ra[2]), "=r"(ra[3]), "=r"(ra[4]), "=r"(ra[5]), "=r"(ra[6]), "=r"(ra[7]),
          "=r"(ra[8]), "=r"(ra[9]), "=r"(ra[10]), "=r"(ra[11]), "=r"(ra[12]), "=r"(ra[13]), "=r"(ra[14]), "=r"(ra[15]),
          "=r"(ra[16]), "=r"(ra[17]), "=r"(ra[18]), "=r"(ra[19]), "=r"(ra[20]), "=r"(ra[21]), "=r"(ra[22]), "=r"(ra[23]),
          "=r"(ra[24]), "=r"(ra[25]), "=r"(ra[26]), "=r"(ra[27]), "=r"(ra[28]), "=r"(ra[29]), "=r"(ra[30]), "=r"(ra[31]),
          "=r"(rb[0]), "=r"(rb[1]), "=r"(rb[2]), "=r"(rb[3]), "=r"(rb[4]), "=r"(rb[5]), "=r"(rb[6]), "=r"(rb[7]),
          "=r"(rb[8]), "=r"(rb[9]), "=r"(rb[10]), "=r"(rb[11]), "=r"(rb[12]), "=r"(rb[13]), "=r"(rb[14]), "=r"(rb[15]),
          "=r"(rb[16]), "=r"(rb[17]), "=r"(rb[18]), "=r"(rb[19]), "=r"(rb[20]), "=r"(rb[21]), "=r"(rb[22]), "=r"(rb[23]),
          "=r"(rb[24]), "=r"(rb[25]), "=r"(rb[26]), "=r"(rb[27]), "=r"(rb[28]), "=r"(rb[29]), "=r"(rb[30]), "=r"(rb[31])
        : "r"(ta), "r"(tb)
        : "memory");
}

// 2^x (approximate, relative error about 2^-22; results below the normal
// range flush to zero, which only drops weights already below 2^-126 of the
// group's largest)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------------------
template <int RATIO, int BN, int COFF = 1>
__global__ void __launch_bounds__(CP_THREADS, 1)
    compressor_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wkv,
                      const __grid_constant__ CUtensorMap tm_wg, const CompressorArgs a) {
    static_assert(BN == 256 || BN == 128, "token tile");
    static_assert(COFF == 1 || (COFF == 2 && RATIO == 4), "the C4A form has cmp_ratio 4");
    // COFF 2: 64 channels per tile, their a and b weight rows interleaved in
    // blocks of 8 (rows 16k .. 16k+7: a channels ch0 + 8k .. +7, rows
    // 16k+8 .. +15: the b channels of the same; one 4-D TMA box per weight
    // and stage), and token tiles overlapping
    // by one 4-token window (each tile starts BN - 4 tokens after the
    // previous one), so that every group's next four tokens sit in its tile
    constexpr int CH_TILE = COFF == 1 ? CP_BM : CP_BM / 2;
    constexpr int TOK_STEP = COFF == 1 ? BN : BN - 4;
    constexpr int CP_STAGES = cp_stages(BN);
    constexpr uint32_t CP_STAGE_BYTES = cp_stage_bytes(BN);
    constexpr uint32_t CP_TMEM_COLS = 2 * BN;          // a power of two >= 32
    constexpr uint32_t CP_GATE_COL = BN;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* tiles = smem_raw + ((1024u - (raw & 1023u)) & 1023u);      // 1024-byte aligned swizzle atoms
    uint64_t* full = reinterpret_cast<uint64_t*>(tiles + CP_STAGES * CP_STAGE_BYTES);
    uint64_t* empty = full + CP_STAGES;
    uint64_t* tmem_full = empty + CP_STAGES;
    uint64_t* tmem_empty = tmem_full + 1;
    uint64_t* drain = tmem_empty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kblocks = a.H / CP_BK;
    const int64_t ntiles = a.n_tok_tiles * a.n_ch_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < CP_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tmem_full, 1);
        mbar_init(tmem_empty, 4 * 32);
        mbar_init(drain, 1);
        mbar_init_fence();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, CP_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            uint32_t it = 0;
            bool dead = false;
            for (int64_t tile = blockIdx.x; tile < ntiles && !dead; tile += gridDim.x) {
                const int32_t tok0 = (int32_t)((tile / a.n_ch_tiles) * TOK_STEP);
                const int32_t ch0 = (int32_t)((tile % a.n_ch_tiles) * CH_TILE);
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const uint32_t st = it % CP_STAGES, round = it / CP_STAGES;
                    if (!mbar_wait_ns(&empty[st], (round & 1u) ^ 1u, CP_WAIT_NS)) {
                        dead = true;
                        break;
                    }
                    uint8_t* s = tiles + st * CP_STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[st], CP_STAGE_BYTES);
                    if (COFF == 1) {
                        tma_load_2d(s, &tm_wkv, kb * CP_BK, ch0, &full[st]);
                        tma_load_2d(s + CP_A_BYTES, &tm_wg, kb * CP_BK, ch0, &full[st]);
                    } else {
                        // the weights seen as [D / 8][2][8][H] (block of 8 channels, a / b
                        // half, row, k): one box of 8 blocks x 2 halves x 8 rows x 64 k
                        // lands rows in the interleaved order 16 block + 8 half + row
                        tma_load_4d(s, &tm_wkv, kb * CP_BK, 0, 0, ch0 / 8, &full[st]);
                        tma_load_4d(s + CP_A_BYTES, &tm_wg, kb * CP_BK, 0, 0, ch0 / 8, &full[st]);
                    }
                    tma_load_2d(s + 2 * CP_A_BYTES, &tm_x, kb * CP_BK, tok0, &full[st]);
                }
            }
            // no load may still be in flight when the CTA exits
            for (uint32_t k = it > CP_STAGES ? it - CP_STAGES : 0; k < it; ++k)
                mbar_wait_ns(&full[k % CP_STAGES], (k / CP_STAGES) & 1u, CP_WAIT_NS);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t IDESC = umma_idesc_bf16(CP_BM, BN);
            uint32_t it = 0, tl = 0;
            bool dead = false;
            for (int64_t tile = blockIdx.x; tile < ntiles && !dead; tile += gridDim.x, ++tl) {
                if (!mbar_wait_ns(tmem_empty, (tl & 1u) ^ 1u, CP_WAIT_NS)) break;   // accumulators free
                tc_fence_after();
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const uint32_t st = it % CP_STAGES, round = it / CP_STAGES;
                    if (!mbar_wait_ns(&full[st], round & 1u, CP_WAIT_NS)) {
                        dead = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t s = smem_u32(tiles + st * CP_STAGE_BYTES);
#pragma unroll
                    for (int k = 0; k < CP_BK / CP_UK; ++k) {
                        const uint64_t dx = umma_desc_sw128(s + 2 * CP_A_BYTES + 32 * k);
                        const uint32_t acc = (kb | k) != 0 ? 1u : 0u;
                        umma_bf16(tmem, umma_desc_sw128(s + 32 * k), dx, IDESC, acc);
                        umma_bf16(tmem + CP_GATE_COL, umma_desc_sw128(s + CP_A_BYTES + 32 * k), dx, IDESC, acc);
                    }
                    umma_commit(&empty[st]);           // the stage is free once these MMAs have read it
                }
                if (!dead) umma_commit(tmem_full);     // the tile's accumulators are complete
            }
            // every MMA issued has completed before TMEM is released
            umma_commit(drain);
            mbar_wait_ns(drain, 0u, CP_WAIT_NS);
        }
    } else {
        // ---------------- epilogue: grouped softmax, Hadamard product, group sum ----------------
        constexpr float LOG2E = 1.4426950408889634f;
        constexpr int R = RATIO < 32 ? RATIO : 32;          // tokens per softmax update
        const int sub = warp & 3;                           // TMEM lane quarter of this warp
        const int row = sub * 32 + lane;                    // channel within the tile
        const uint32_t tbase = tmem + ((uint32_t)(sub * 32) << 16);
        uint32_t tl = 0;
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tl) {
            const int64_t tok0 = (tile / a.n_ch_tiles) * TOK_STEP;
            if (!__all_sync(FULL_MASK, mbar_wait_ns(tmem_full, tl & 1u, CP_WAIT_NS))) break;
            tc_fence_after();
            if (COFF == 2) {
                // lane l and l ^ 8 hold the a and b rows of one channel.  In every
                // 4-token window both lanes reduce their own four rows (softmax
                // maximum, weight sum, weighted kv sum): the a lane those of the
                // group that the window opens, the b lane the next-window half of
                // the group that the window closes; the b lane's three values then
                // cross to the a lane, which merges them with the a part it kept
                // from the previous window and writes the closed group.
                const bool is_a = (row & 8) == 0;
                const int ch = (int)((tile % a.n_ch_tiles) * CH_TILE) + 8 * (row >> 4) + (row & 7);
                float ap[4];                                       // this lane's Ape column, rows of 2 D
#pragma unroll
                for (int i = 0; i < 4; ++i) ap[i] = __ldg(a.ape + (int64_t)i * 2 * a.D + (is_a ? 0 : a.D) + ch);
                float pm = 0.0f, pl = 0.0f, pacc = 0.0f;            // the open group's a part (a lanes)
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    if (tok0 + c0 >= a.T) break;                   // past the chunk (warp-uniform)
                    uint32_t kv[32], gs[32];
                    tmem_ld32x2(tbase + (uint32_t)c0, tbase + CP_GATE_COL + (uint32_t)c0, kv, gs);
#pragma unroll
                    for (int w = 0; w < 8; ++w) {
                        const int u = c0 / 4 + w;                  // window within the tile
                        const int64_t t4 = tok0 + 4 * u;           // its first token
                        if (t4 >= a.T) break;                      // warp-uniform
                        float sc[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) sc[i] = __fadd_rn(__uint_as_float(gs[4 * w + i]), ap[i]);
                        const float cm = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
                        float l = 0.0f, acc = 0.0f;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float p = ex2_approx(__fmul_rn(__fsub_rn(sc[i], cm), LOG2E));
                            l = __fadd_rn(l, p);
                            acc = __fmaf_rn(p, __uint_as_float(kv[4 * w + i]), acc);
                        }
                        const float om = __shfl_xor_sync(FULL_MASK, cm, 8);
                        const float ol = __shfl_xor_sync(FULL_MASK, l, 8);
                        const float oacc = __shfl_xor_sync(FULL_MASK, acc, 8);
                        if (!is_a) continue;
                        if (u > 0) {
                            // close the group of window u - 1: its a part and this window's b part
                            const float mn = fmaxf(pm, om);
                            const float ca = ex2_approx(__fmul_rn(__fsub_rn(pm, mn), LOG2E));
                            const float cb = ex2_approx(__fmul_rn(__fsub_rn(om, mn), LOG2E));
                            const float L = __fmaf_rn(ol, cb, __fmul_rn(pl, ca));
                            const float A = __fmaf_rn(oacc, cb, __fmul_rn(pacc, ca));
                            a.out[(t4 / 4 - 1) * a.D + ch] = (uint16_t)to_bf16_bits(__fdiv_rn(A, L));
                        }
                        if (u < BN / 4 - 1) {
                            if (t4 + 4 >= a.T)                     // the last group: no next four tokens
                                a.out[(t4 / 4) * a.D + ch] = (uint16_t)to_bf16_bits(__fdiv_rn(acc, l));
                            pm = cm;
                            pl = l;
                            pacc = acc;
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(tmem_empty);
                continue;
            }
            const int ch = (int)((tile % a.n_ch_tiles) * CP_BM) + row;
            float m = -INFINITY, l = 0.0f, acc = 0.0f;
            for (int c0 = 0; c0 < BN; c0 += 32) {
                if (tok0 + c0 >= a.T) break;                 // ragged last tile (warp-uniform)
                uint32_t kv[32], gs[32];
                tmem_ld32x2(tbase + (uint32_t)c0, tbase + CP_GATE_COL + (uint32_t)c0, kv, gs);
#pragma unroll
                for (int s0 = 0; s0 < 32; s0 += R) {
                    if (tok0 + c0 + s0 >= a.T) break;
                    float sc[R];
                    float cm = -INFINITY;
#pragma unroll
                    for (int i = 0; i < R; ++i) {
                        const int pos = (c0 + s0 + i) % RATIO;                 // token position in its group
                        sc[i] = __fadd_rn(__uint_as_float(gs[s0 + i]), __ldg(a.ape + (int64_t)pos * a.D + ch));
                        cm = fmaxf(cm, sc[i]);
                    }
                    const float mn = fmaxf(m, cm);
                    const float corr = ex2_approx(__fmul_rn(__fsub_rn(m, mn), LOG2E));   // 0 for the first update
                    l = __fmul_rn(l, corr);
                    acc = __fmul_rn(acc, corr);
#pragma unroll
                    for (int i = 0; i < R; ++i) {
                        const float p = ex2_approx(__fmul_rn(__fsub_rn(sc[i], mn), LOG2E));
                        l = __fadd_rn(l, p);
                        acc = __fmaf_rn(p, __uint_as_float(kv[s0 + i]), acc);
                    }
                    m = mn;
                    if ((c0 + s0 + R) % RATIO == 0) {
                        const int64_t g = (tok0 + c0 + s0 + R) / RATIO - 1;
                        a.out[g * a.D + ch] = (uint16_t)to_bf16_bits(__fdiv_rn(acc, l));
                        m = -INFINITY;
                        l = 0.0f;
                        acc = 0.0f;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(tmem_empty);                         // this thread is done with the accumulators
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, CP_TMEM_COLS);
    }
}

}  // namespace kvq
