"""CUDA library vs the CPU oracle, byte for byte, through the C ABI.

Every comparison covers the cache's whole byte storage (guard bands, block
padding, headDim tails, skipped and unmapped rows included).  Small cases span
several warp tiles and a ragged tail; the five named workloads run at full size.
"""
import numpy as np
import pytest
import torch

import kv_cache_quantize_b200 as kvq
import oracle
from _gpu_harness import run_gpu
from _oracle_harness import run_oracle
from kv_cache_quantize_b200 import workloads as W

pytestmark = pytest.mark.gpu
THREADS = 16


def _same(case, check_outputs=True, misalign=False):
    st_o, out_o, f_o = run_oracle(case, threads=THREADS)
    st_g, out_g, f_g = run_gpu(case, misalign)
    assert f_g == f_o, f"fault bits gpu={f_g} oracle={f_o}"
    for k in st_o:
        a, b = st_g[k], st_o[k]
        bad = np.nonzero(a != b)[0]
        assert bad.size == 0, f"{case.name}/{k}: {bad.size} bytes differ, first at {bad[0]} gpu={a[bad[0]]:#x} oracle={b[bad[0]]:#x}"
    if check_outputs:
        for k, v in out_o.items():
            if v is None:
                continue
            g = out_g[k].reshape(v.shape)
            bad = np.nonzero(g != v)[0] if g.ndim == 1 else np.argwhere(g != v)
            assert len(bad) == 0, f"{case.name}/{k}: {len(bad)} values differ"
    return st_g, out_g


# ---------------------------------------------------------------------------
# kv_compress_epilog
# ---------------------------------------------------------------------------
def _ce(T, d, mode, G=64, kind="normal", pad=0, extra=13, skip=0.1, seed=0, slot_dtype=np.int32, xs=0.1,
        block_size=16, x_dtype="bf16"):
    col = oracle.kv_cache_col(d, mode, G)
    nblk = max(1, (2 * T + block_size - 1) // block_size)
    return W.gen_compress(f"ce_m{mode}_g{G}_d{d}_T{T}_{kind}_{x_dtype}", T=T, d=d, quant_mode=mode,
                          num_blocks=nblk, block_size=block_size, head_dim=col + extra, group_size=G, x_scale=xs,
                          skip_frac=skip, outlier_frac=0.05, seed=seed, x_kind=kind, block_pad_bytes=pad,
                          slot_dtype=slot_dtype, x_dtype=x_dtype)


@pytest.mark.parametrize("kind", ["normal", "wide"])
@pytest.mark.parametrize("mode,G", [(0, 64), (1, 64), (2, 16), (2, 32), (2, 64)])
@pytest.mark.parametrize("d", [128, 576, 1024])
def test_compress_small(mode, G, d, kind):
    _same(_ce(203, d, mode, G, kind))


@pytest.mark.parametrize("mode,G", [(0, 64), (1, 64), (2, 32)])
@pytest.mark.parametrize("extra,pad", [(0, 0), (1, 0), (3, 40), (16, 1000), (7, 5)])
def test_compress_row_alignments(mode, G, extra, pad):
    """headDim tails and block strides that make rows start at every alignment."""
    _same(_ce(77, 320, mode, G, extra=extra, pad=pad, seed=5))


@pytest.mark.parametrize("T", [0, 1, 7, 8, 9, 31, 33])
def test_compress_ragged_counts(T):
    _same(_ce(T, 576, 0, seed=7))


# Batches of at least one 32-row tile per SM take the pipelined (bulk-copy)
# kernel; smaller ones the direct kernel.  T_PIPE is above that threshold on
# any GPU with up to 188 SMs and leaves a ragged last tile.
T_PIPE = 6037


@pytest.mark.parametrize("mode,G", [(0, 64), (1, 64), (2, 16), (2, 32), (2, 64)])
@pytest.mark.parametrize("d", [128, 576, 1024])
def test_compress_pipelined(mode, G, d):
    _same(_ce(T_PIPE, d, mode, G, kind="wide" if d == 576 else "normal", seed=21))


@pytest.mark.parametrize("mode,G", [(0, 64), (1, 64), (2, 32)])
@pytest.mark.parametrize("extra,pad", [(0, 0), (1, 0), (3, 40), (16, 1000)])
def test_compress_pipelined_row_alignments(mode, G, extra, pad):
    _same(_ce(T_PIPE, 320, mode, G, extra=extra, pad=pad, seed=23))


@pytest.mark.parametrize("T", [6016, 6017, 6047])
def test_compress_pipelined_ragged_counts(T):
    _same(_ce(T, 576, 2, 32, seed=25))


# d > 1024: more 64-value segment columns (17, 22, 27) than the pipelined
# kernel's 16 consumer warps, so each warp walks several columns and packed
# rows leave by direct stores; 1728 is the widest row whose two-stage ring
# fits in shared memory.
@pytest.mark.parametrize("mode,G", [(0, 64), (1, 64), (2, 16), (2, 32), (2, 64)])
@pytest.mark.parametrize("d", [1088, 1408, 1728])
def test_compress_pipelined_multi_segment_columns(mode, G, d):
    _same(_ce(T_PIPE, d, mode, G, kind="wide" if d == 1408 else "normal", seed=31))


@pytest.mark.parametrize("mode,G", [(0, 64), (1, 64), (2, 16)])
@pytest.mark.parametrize("extra,pad", [(1, 0), (7, 5), (16, 1000)])
def test_compress_pipelined_multi_segment_row_alignments(mode, G, extra, pad):
    _same(_ce(T_PIPE, 1408, mode, G, extra=extra, pad=pad, seed=33))


@pytest.mark.parametrize("mode,G", [(0, 64), (1, 64), (2, 16), (2, 64)])
def test_compress_widest_rows_at_pipelined_batch_size(mode, G):
    """d = 8192 with a batch above the pipelined threshold: the ring does not fit
    in shared memory, so kernel selection must fall back to the direct kernel."""
    _same(_ce(T_PIPE, 8192, mode, G, seed=35, slot_dtype=np.int64 if mode == 0 else np.int32))


def test_compress_max_width_and_int64_slots():
    _same(_ce(40, 8192, 0, seed=9, slot_dtype=np.int64))
    _same(_ce(40, 8192, 2, 16, seed=9, slot_dtype=np.int64))
    _same(_ce(40, 8192, 1, seed=9))


def test_compress_strided_and_misaligned_x():
    case = _ce(50, 256, 0, seed=11)
    st_o, _, _ = run_oracle(case)
    x = case.arrays["x"]
    dev = "cuda"
    # rows 320 elements apart (non-contiguous leading dim), and a view starting 1 element in
    for stride_extra, shift in ((64, 0), (0, 1), (3, 1)):
        row = x.shape[1] + stride_extra
        buf = np.zeros(x.shape[0] * row + shift + 8, dtype=np.uint16)
        for t in range(x.shape[0]):
            buf[shift + t * row: shift + t * row + x.shape[1]] = x[t]
        tb = torch.from_numpy(buf.view(np.int16)).view(torch.bfloat16).to(dev)
        xv = tb[shift:shift + x.shape[0] * row].view(x.shape[0], row)[:, :x.shape[1]]
        cb = case.caches["cache"]
        st = torch.from_numpy(cb.storage.copy()).to(dev)
        view = st[cb.offset:].as_strided((cb.num_blocks, cb.block_size, 1, cb.head_dim),
                                         (cb.block_stride, cb.head_dim, cb.head_dim, 1))
        kvq.kv_compress_epilog(xv, torch.from_numpy(case.arrays["slot_mapping"]).to(dev), view, 0)
        torch.cuda.synchronize()
        assert np.array_equal(st.cpu().numpy(), st_o["cache"]), (stride_extra, shift)


def test_compress_bad_slots_raise_fault_and_skip():
    case = _ce(64, 576, 0, seed=13)
    s = case.arrays["slot_mapping"]
    s[3] = case.caches["cache"].num_slots
    s[10] = -5
    s[11:20] = -1
    _same(case)


def test_compress_all_skipped():
    case = _ce(64, 576, 2, 32, seed=15)
    case.arrays["slot_mapping"][:] = -1
    st_g, _ = _same(case)
    assert np.array_equal(st_g["cache"], case.caches["cache"].storage)


# float16 x (quantMode 0/1: the page requires bfloat16 only in mode 2), on the
# direct kernel (decode-sized batches, misaligned rows) and the pipelined one
@pytest.mark.parametrize("kind", ["normal", "wide"])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("T,d", [(203, 576), (T_PIPE, 576), (T_PIPE, 1408), (45, 8192)])
def test_compress_f16_x(mode, T, d, kind):
    _same(_ce(T, d, mode, kind=kind, seed=43, x_dtype="f16"))


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("extra,pad", [(1, 0), (3, 40)])
def test_compress_f16_x_row_alignments(mode, extra, pad):
    _same(_ce(T_PIPE, 320, mode, extra=extra, pad=pad, seed=45, x_dtype="f16"))


@pytest.mark.parametrize("name", ["compress_mode1_T64_d256", "compress_mode0_T262144_d576",
                                  "compress_mode2_G32_T262144_d576", "compress_mode0_f16_T262144_d576"])
def test_compress_named_workloads_full_size(name):
    _same(W.CONFIGS[name]())


def test_compress_is_deterministic():
    case = W.compress_mode2_G32_T262144_d576()
    a, _, _ = run_gpu(case)
    b, _, _ = run_gpu(case)
    assert np.array_equal(a["cache"], b["cache"])


# ---------------------------------------------------------------------------
# indexer_quant_cache
# ---------------------------------------------------------------------------
def _ix(T, d, mode, cdt="e4m3", xdt="bf16", kind="student_t", pad=0, seed=0, extra=5):
    scol = oracle.indexer_scale_col(d, mode)
    code_bytes = (d + 1) // 2 if mode == 3 else d
    return W.gen_indexer(f"ix_m{mode}_{cdt}_{xdt}_d{d}_T{T}", T=T, d=d, quant_mode=mode,
                         num_blocks=max(1, (2 * T + 7) // 8), block_size=8, cache_head_dim=code_bytes + extra,
                         scale_head_dim=scol + 3, cache_dtype=cdt, x_dtype=xdt, skip_frac=0.1, seed=seed,
                         block_pad_bytes=pad, x_kind=kind)


@pytest.mark.parametrize("xdt", ["bf16", "f16"])
@pytest.mark.parametrize("mode,cdt", [(0, "e4m3"), (0, "e5m2"), (1, "e4m3"), (1, "e5m2"), (3, "u8")])
@pytest.mark.parametrize("d", [32, 99, 128, 200, 256, 520])
def test_indexer_small(mode, cdt, d, xdt):
    _same(_ix(150, d, mode, cdt, xdt, seed=d))


@pytest.mark.parametrize("mode,cdt", [(0, "e4m3"), (1, "e5m2"), (3, "u8")])
def test_indexer_wide_values_and_padding(mode, cdt):
    _same(_ix(97, 128, mode, cdt, kind="wide", pad=24, extra=0, seed=3))


@pytest.mark.parametrize("name", ["indexer_mxfp8_T65536_d128", "indexer_mxfp4_T65536_d128", "indexer_fp8_T65536_d128",
                                  "indexer_mxfp8_e5m2_T65536_d128"])
def test_indexer_named_workloads_full_size(name):
    _same(W.CONFIGS[name]())


def test_indexer_bad_slot_fault():
    case = _ix(64, 128, 0)
    case.arrays["slot_mapping"][5] = case.caches["cache"].num_slots + 3
    _same(case)


# ---------------------------------------------------------------------------
# kv_rmsnorm_rope_cache
# ---------------------------------------------------------------------------
def _rr(cache_mode="PA_BNSD", B=40, S=1, k_dtype="bf16", ckv_dtype="e4m3", kv_dtype="bf16", D=576, Dv=512,
        seed=0, block_size=32, **kw):
    opt = {"block_pad_bytes": 64}
    if ckv_dtype in ("e4m3", "e5m2", "i8"):
        opt["ckv_scale"] = [1 / 64]
    if k_dtype in ("e4m3", "e5m2", "i8"):
        opt["k_scale"] = [1 / 16]
    if ckv_dtype == "i8":
        opt["ckv_offset"] = [2.0]
    opt.update(kw)
    return W.gen_rmsnorm_rope(f"rr_{cache_mode}_{k_dtype}_{ckv_dtype}_{kv_dtype}_D{D}", B=B, S=S, D=D, Dv=Dv,
                              num_blocks=max(B + 1, (2 * B * S) // block_size + 2), block_size=block_size,
                              k_dtype=k_dtype,
                              ckv_dtype=ckv_dtype, cache_mode=cache_mode, skip_frac=0.1, seed=seed,
                              kv_dtype=kv_dtype, **opt)


@pytest.mark.parametrize("cache_mode,S", [("PA_BNSD", 1), ("PA", 3), ("Norm", 5), ("PA_BLK_BNSD", 70)])
def test_rmsnorm_rope_cache_modes(cache_mode, S):
    _same(_rr(cache_mode, B=6 if S > 1 else 40, S=S))


@pytest.mark.parametrize("k_dtype,ckv_dtype", [("bf16", "bf16"), ("bf16", "e4m3"), ("f16", "e5m2"),
                                               ("bf16", "i8"), ("e4m3", "bf16"), ("i8", "f16"),
                                               ("e4m3", "e4m3"), ("i8", "i8")])
def test_rmsnorm_rope_dtype_scenarios(k_dtype, ckv_dtype):
    _same(_rr(k_dtype=k_dtype, ckv_dtype=ckv_dtype))


@pytest.mark.parametrize("D,Dv", [(192, 128), (96, 32), (1034, 1000)])
def test_rmsnorm_rope_other_widths_and_f16(D, Dv):
    _same(_rr(D=D, Dv=Dv, kv_dtype="f16", k_dtype="f16", ckv_dtype="f16"))
    _same(_rr(D=D, Dv=Dv))


def test_rmsnorm_rope_named_workload_full_size():
    _same(W.rmsnorm_rope_decode_B64_D576())


@pytest.mark.parametrize("name", ["rmsnorm_rope_prefill_B65536_D576", "rmsnorm_rope_int8_prefill_B65536_D576"])
def test_rmsnorm_rope_prefill_size(name):
    _same(W.CONFIGS[name]())


@pytest.mark.parametrize("ckv_dtype", ["bf16", "e4m3"])
def test_rmsnorm_rope_subnormal_and_tie_quotients(ckv_dtype):
    """Rows whose x / rms quotients are subnormal, two of them exact rounding
    ties (epsilon 0): rms = 2^17 with x = 3 * 2^-133 (quotient 3 * 2^-150,
    which rounds to the even 2^-148) and rms = 3 * 2^17 with the same x
    (quotient 2^-150, which rounds to 0); other rows mix bf16 subnormals, zeros
    and large values into random rows."""
    case = _rr(B=48, ckv_dtype=ckv_dtype, k_dtype="bf16", seed=41, epsilon=0.0)
    kv = case.arrays["kv"].reshape(48, 576)
    live = np.nonzero(case.arrays["index"].reshape(-1) != -1)[0]
    bits = lambda v: W.to_bf16_bits(np.array([v], dtype=np.float32))[0]
    for r, big in ((live[0], 2.0 ** 21), (live[1], 3.0 * 2.0 ** 21)):
        kv[r, :512] = 0
        kv[r, 10] = kv[r, 300] = bits(big)
        kv[r, 77] = 3                                 # 3 * 2^-133, a bf16 subnormal
        kv[r, 78] = 3 | 0x8000                        # its negative
    # a gamma of 2^100 on those two channels carries the quotients' last bits
    # into the output (2^-148 * 2^100 = 2^-48 is a normal bf16 value)
    case.arrays["gamma"][77] = case.arrays["gamma"][78] = bits(2.0 ** 100)
    rng = np.random.default_rng(43)
    for r in live[2::3]:
        cols = rng.choice(512, size=12, replace=False)
        sign = (rng.integers(0, 2, size=6) << 15).astype(np.uint16)
        kv[r, cols[:6]] = rng.integers(1, 128, size=6).astype(np.uint16) | sign
        kv[r, cols[6:9]] = 0
        kv[r, cols[9:]] = bits(2.0 ** 40)
    _same(case)


# The lean kernel takes Dv of 256, 512 or 1024 with Dk = 64, PA / PA_BNSD,
# cache rows aligned for whole-chunk stores; the cases below reach each of its
# template instances at a decode-sized and a prefill-sized batch (4803 tokens,
# several per warp), and the per-tensor FP8 scale forms.
@pytest.mark.parametrize("B", [70, 4803])
@pytest.mark.parametrize("kv_dtype", ["bf16", "f16"])
@pytest.mark.parametrize("D,Dv", [(320, 256), (576, 512), (1088, 1024)])
def test_rmsnorm_rope_lean_shapes(D, Dv, kv_dtype, B):
    for i, (k_dtype, ckv_dtype) in enumerate([(kv_dtype, kv_dtype), (kv_dtype, "e4m3"), (kv_dtype, "e5m2"),
                                              ("i8", "i8"), ("e5m2", "e5m2")]):
        _same(_rr("PA" if i % 2 else "PA_BNSD", B=B, S=1, D=D, Dv=Dv, kv_dtype=kv_dtype, k_dtype=k_dtype,
                  ckv_dtype=ckv_dtype, seed=100 + i, slot_dtype=np.int64 if i == 3 else np.int32))


@pytest.mark.parametrize("scale", [1 / 64, 0.013, "per_channel"])
def test_rmsnorm_rope_ring_fp8_scales_and_unaligned_rope(scale):
    """Prefill-sized batches with the folded and the separate FP8 scale
    forms, with cos / sin 16-byte aligned and one element past a 16-byte
    boundary."""
    kw = {"ckv_scale": (2.0 ** np.random.default_rng(3).integers(-8, 0, 512)).tolist()
          if scale == "per_channel" else [scale]}
    case = _rr(B=4803, ckv_dtype="e4m3", seed=71, **kw)
    _same(case)
    _same(case, misalign=True)


@pytest.mark.parametrize("ckv_dtype", ["e4m3", "e5m2"])
@pytest.mark.parametrize("scale", [1 / 64, 2.0 ** -109, 2.0 ** -110, 1.0, 8.0, 0.013, "per_channel", "big_gamma"])
def test_rmsnorm_rope_fp8_scale_forms(ckv_dtype, scale):
    """The per-tensor power-of-two scales 2^-k with 0 <= k <= 109 fold into the
    staged gamma; 2^-110, 8 (k < 0), a scale that is not a power of two, a
    per-channel scale, and a gamma whose product with 64 overflows take the
    separate forms."""
    kw = {}
    if scale == "per_channel":
        kw["ckv_scale"] = (2.0 ** np.random.default_rng(3).integers(-8, 0, 512)).tolist()
    elif scale == "big_gamma":
        kw["ckv_scale"] = [1 / 64]
    else:
        kw["ckv_scale"] = [scale]
    case = _rr(B=64, ckv_dtype=ckv_dtype, seed=61, **kw)
    if scale == "big_gamma":
        case.arrays["gamma"][[5, 300]] = W.to_bf16_bits(np.array([2.0 ** 126, -3.0 * 2.0 ** 125], np.float32))
    _same(case)


@pytest.mark.parametrize("ckv_dtype,pad", [("e4m3", 8), ("bf16", 8), ("e4m3", 4), ("bf16", 2)])
def test_rmsnorm_rope_cache_row_alignment(ckv_dtype, pad):
    """Cache blocks padded so that rows are 8-, 4- or 2-byte aligned only:
    the lean kernel takes the 8-aligned FP8 cache, the general kernel the
    rest."""
    _same(_rr(B=60, ckv_dtype=ckv_dtype, seed=67, block_pad_bytes=pad))


@pytest.mark.parametrize("ckv_dtype,block_size", [("bf16", 48), ("e4m3", 96)])
@pytest.mark.parametrize("B", [70, 4803])
def test_rmsnorm_rope_block_size_not_power_of_two(ckv_dtype, block_size, B):
    """Slots map to (block, row) by division when blockSize is not a power of
    two (48 for 16-bit caches, 96 for a 1-byte ckv cache: the page's multiples
    of 16 and 32)."""
    _same(_rr(B=B, ckv_dtype=ckv_dtype, seed=73, block_size=block_size))


@pytest.mark.parametrize("D,Dv,cache_mode", [(576, 512, "PA_BNSD"), (576, 512, "PA"), (192, 128, "PA_BNSD")])
@pytest.mark.parametrize("slot_dtype", [np.int32, np.int64])
def test_rmsnorm_rope_bad_index_fault(D, Dv, cache_mode, slot_dtype):
    """Index entries past the cache, negative ones other than -1, and (int64)
    one at 2^31: each such token is skipped and the fault bit is raised, as
    the oracle does."""
    case = _rr(cache_mode, B=60, D=D, Dv=Dv, seed=79, slot_dtype=slot_dtype)
    idx = case.arrays["index"].reshape(-1)
    n = case.caches["k_cache"].num_slots
    idx[5] = n
    idx[17] = -7
    if slot_dtype == np.int64:
        idx[31] = 2 ** 31
    _same(case)


@pytest.mark.parametrize("ckv_dtype", ["bf16", "e4m3", "i8"])
def test_rmsnorm_rope_tiny_rows(ckv_dtype):
    """Rows of tiny values (epsilon 0), so that the squares are subnormal
    binary32 numbers: bf16 exponent fields drawn from [50, 59] (|x| < 2^-67,
    x * x not exact in binary32), from [60, 70] (x * x exact), or both mixed
    in one row; the sum of squares must match the separately rounded
    RN(acc + RN(x * x)) of the page's formula either way."""
    case = _rr(B=48, ckv_dtype=ckv_dtype, k_dtype="bf16", seed=47, epsilon=0.0)
    kv = case.arrays["kv"].reshape(48, 576)
    rng = np.random.default_rng(53)
    for r in range(48):
        lo, hi = ((50, 59), (60, 70), (50, 70))[r % 3]
        e = rng.integers(lo, hi + 1, size=512).astype(np.uint16)
        m = rng.integers(0, 128, size=512).astype(np.uint16)
        sign = (rng.integers(0, 2, size=512) << 15).astype(np.uint16)
        kv[r, :512] = sign | (e << 7) | m
    _same(case)


@pytest.mark.parametrize("ckv_dtype,k_dtype", [("i8", "bf16"), ("bf16", "bf16"), ("e5m2", "f16"), ("i8", "i8")])
def test_rmsnorm_rope_vector_path_dtypes(ckv_dtype, k_dtype):
    """Aligned rows with Dv = 256 / 512 / 1024 take the register-chunk kernel for every ckv dtype."""
    for D, Dv in ((320, 256), (576, 512), (1088, 1024)):
        _same(_rr(D=D, Dv=Dv, k_dtype=k_dtype, ckv_dtype=ckv_dtype))


# ---------------------------------------------------------------------------
# dequant_rope_quant_kvcache
# ---------------------------------------------------------------------------
def _dq(**kw):
    base = dict(B=3, S=40, Nq=4, Nkv=2, D=128, c0=8, c1=64, x_range=1 << 12, seed=1, block_pad_bytes=40)
    base.update(kw)
    name = "dq_" + "_".join(f"{k}{v}" for k, v in sorted(kw.items()))
    return W.gen_dequant_rope_quant(name, **base)


@pytest.mark.parametrize("cache_mode", ["page", "contiguous"])
@pytest.mark.parametrize("kv_output", [False, True])
def test_drq_modes(cache_mode, kv_output):
    _same(_dq(cache_mode=cache_mode, kv_output=kv_output, skip_frac=0.1 if cache_mode == "page" else 0.0))


@pytest.mark.parametrize("D", [32, 64, 96, 256])
def test_drq_head_dims(D):
    _same(_dq(D=D, Nq=4, Nkv=1, kv_output=True))   # H = 6*D, a multiple of 64


# head sizes a multiple of 16 but not of 32 (pipelined kernel, D/8 lanes per
# head), and heads wider than 256 (general kernel); H = 4 D a multiple of 64
@pytest.mark.parametrize("D", [16, 48, 80, 512, 1024])
def test_drq_other_head_dims(D):
    _same(_dq(D=D, Nq=2, Nkv=1, kv_output=True, S=12))


# inputs off 16-byte alignment take the general kernel
@pytest.mark.parametrize("D,x_dtype", [(128, "i32"), (64, "bf16"), (16, "i32"), (512, "f16")])
@pytest.mark.parametrize("cache_mode", ["page", "contiguous"])
def test_drq_unaligned_inputs(D, x_dtype, cache_mode):
    _same(_dq(D=D, Nq=2, Nkv=1, S=12, x_dtype=x_dtype, cos_dtype="bf16" if x_dtype != "f16" else "f16",
              kv_output=True, cache_mode=cache_mode, skip_frac=0.1 if cache_mode == "page" else 0.0),
          misalign=True)


def test_drq_unaligned_bias_kinds_and_named_shape():
    for bias_dtype in ("bf16", "i32", None):
        _same(_dq(bias_dtype=bias_dtype, with_offsets=bias_dtype is not None,
                  with_activation_scale=bias_dtype is not None), misalign=True)
    _same(W.dequant_rope_quant_page_B16_S1024_H3072(x_range=1 << 12), misalign=True)


@pytest.mark.parametrize("bias_dtype", ["f32", "bf16", "f16", "i32", None])
def test_drq_bias_and_optional_inputs(bias_dtype):
    _same(_dq(bias_dtype=bias_dtype, with_offsets=bias_dtype is not None,
              with_activation_scale=bias_dtype != "f16"))


@pytest.mark.parametrize("x_dtype", ["bf16", "f16"])
def test_drq_float_input(x_dtype):
    _same(_dq(x_dtype=x_dtype, cos_dtype=x_dtype, kv_output=True))


def test_drq_two_dim_x():
    _same(_dq(S=1, x_2d=True, kv_output=True, cache_mode="contiguous"))


@pytest.mark.parametrize("B", [1, 97])
def test_drq_operator_test_suite_shapes(B):
    """The two end-to-end cases of the operator's own test suite
    (aclnnDequantRopeQuantKvcache, 测试与验证): 2-D x [1, 2304] float16 split
    1536/384/384, and 2-D x [1, 3584] int32 split 1792/896/896 with a bf16
    bias, both in page mode.  The page gives the splits, not the head size:
    D = 128 (so Nq, Nkv = 12, 3 and 14, 7).  B = 97 repeats each shape over
    more rows."""
    _same(_dq(B=B, S=1, x_2d=True, Nq=12, Nkv=3, D=128, x_dtype="f16", cos_dtype="f16", cache_mode="page",
              c0=4, c1=64, kv_output=True))
    _same(_dq(B=B, S=1, x_2d=True, Nq=14, Nkv=7, D=128, bias_dtype="bf16", cache_mode="page", c0=4, c1=64))


def test_drq_many_heads():
    _same(_dq(Nq=40, Nkv=8, D=32, S=8))


def test_drq_bad_index_fault():
    case = _dq(cache_mode="page")
    case.arrays["indices"][7] = case.caches["k_cache"].num_slots
    _same(case)


@pytest.mark.parametrize("name", ["dequant_rope_quant_page_B16_S1024_H3072",
                                  "dequant_rope_quant_contiguous_kvout_B16_S1024_H3072",
                                  "dequant_rope_quant_bf16_page_B16_S1024_H3072"])
def test_drq_named_workload_full_size(name):
    _same(W.CONFIGS[name]())


def test_drq_named_workload_narrow_range():
    """Same shapes with |x| <= 2^12, where few int8 codes saturate."""
    _same(W.dequant_rope_quant_page_B16_S1024_H3072(x_range=1 << 12))


# ---------------------------------------------------------------------------
# scatter_rows: the compress access pattern without arithmetic (data movement
# only, so the expectation is the input bytes themselves)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("out_bytes", [352, 672, 1152])
def test_scatter_rows_moves_the_row_prefix(out_bytes):
    from kv_cache_quantize_b200.workloads import dev_cache
    case = _ce(T_PIPE, 576, 0, seed=41, extra=1152 - oracle.kv_cache_col(576, 0, 64))
    x, slots, cb = case.arrays["x"], case.arrays["slot_mapping"], case.caches["cache"]
    st, view = dev_cache(cb, torch.uint8)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    kvq.get_error()
    kvq.scatter_rows(xt, torch.from_numpy(slots).cuda(), view, out_bytes)
    torch.cuda.synchronize()
    assert kvq.get_error() == 0
    want = cb.storage.copy()
    xb = x.view(np.uint8).reshape(x.shape[0], -1)
    for t, s in enumerate(slots.tolist()):
        if s >= 0:
            o = cb.offset + (s // cb.block_size) * cb.block_stride + (s % cb.block_size) * cb.row_bytes
            want[o:o + out_bytes] = xb[t, :out_bytes]
    assert np.array_equal(st.cpu().numpy(), want)
