"""Packed-row decoder: CUDA library vs the CPU oracle, bit for bit, through the
C ABI.  The packed caches are written by the oracle's encoder (so the decoder
is checked on its own), then both decoders read them into y buffers pre-filled
with a marker, which also checks that rows of skipped tokens stay untouched.
"""
import numpy as np
import pytest
import torch

import kv_cache_quantize_b200 as kvq
import oracle
from _oracle_harness import paged
from kv_cache_quantize_b200 import workloads as W

pytestmark = pytest.mark.gpu
THREADS = 16
MARK = 0x7E57


def _encoded(case):
    st = case.caches["cache"].storage.copy()
    a, at = case.arrays, case.attrs
    oracle.kv_compress_epilog(a["x"], a["slot_mapping"], paged(case.caches["cache"], st), at["quant_mode"],
                              at["quant_group_size"], at["x_scale"], THREADS, x_dtype=at.get("x_dtype", "bf16"))
    return st


def _same(case, slots=None, y_extra=0, y_shift=0):
    at = case.attrs
    cb = case.caches["cache"]
    st = _encoded(case)
    slots = case.arrays["slot_mapping"] if slots is None else slots
    T, d = case.arrays["x"].shape
    mode, G, xs = at["quant_mode"], at["quant_group_size"], at["x_scale"]
    ydt = at.get("x_dtype", "bf16")
    y_o, f_o = oracle.kv_decompress(paged(cb, st.copy()), slots, d, mode, G, xs,
                                    y=np.full((T, d), MARK, dtype=np.uint16), threads=THREADS, y_dtype=ydt)
    # device: the same packed bytes; y rows possibly strided / shifted
    dst = torch.from_numpy(st).cuda()
    view = dst[cb.offset:].as_strided((cb.num_blocks, cb.block_size, 1, cb.head_dim),
                                      (cb.block_stride, cb.head_dim, cb.head_dim, 1))
    row = d + y_extra
    buf = torch.full((T * row + y_shift + 16,), MARK, dtype=torch.int16, device="cuda")
    y = buf[y_shift:y_shift + T * row].view(T, row)[:, :d].view(torch.bfloat16 if ydt == "bf16" else torch.float16)
    kvq.get_error()
    kvq.kv_decompress(view, torch.from_numpy(np.ascontiguousarray(slots)).cuda(), y, mode, G, xs)
    torch.cuda.synchronize()
    f_g = kvq.get_error()
    y_g = y.view(torch.int16).cpu().numpy().view(np.uint16)
    assert f_g == f_o
    bad = np.argwhere(y_g != y_o)
    assert len(bad) == 0, f"{case.name}: {len(bad)} values differ, first {bad[0]} gpu={y_g[tuple(bad[0])]:#x} " \
                          f"oracle={y_o[tuple(bad[0])]:#x}"
    # the device must not have written outside y's rows
    rest = buf.cpu().numpy().view(np.uint16)
    mask = np.ones(rest.size, dtype=bool)
    for t in range(T):
        mask[y_shift + t * row: y_shift + t * row + d] = False
    assert np.all(rest[mask] == MARK)
    return y_g


def _case(T, d, mode, G=64, kind="normal", extra=13, pad=0, seed=0, skip=0.1, slot_dtype=np.int32, xs=0.1,
          x_dtype="bf16"):
    col = oracle.kv_cache_col(d, mode, G)
    nblk = max(1, (2 * T + 15) // 16)
    return W.gen_compress(f"kd_m{mode}_g{G}_d{d}_T{T}_{kind}_{x_dtype}", T=T, d=d, quant_mode=mode,
                          num_blocks=nblk, block_size=16, head_dim=col + extra, group_size=G, x_scale=xs,
                          skip_frac=skip, outlier_frac=0.05, seed=seed, x_kind=kind, block_pad_bytes=pad,
                          slot_dtype=slot_dtype, x_dtype=x_dtype)


@pytest.mark.parametrize("kind", ["normal", "wide"])
@pytest.mark.parametrize("mode,G", [(0, 64), (1, 64), (2, 16), (2, 32), (2, 64)])
@pytest.mark.parametrize("d", [128, 320, 576, 832, 1024])
def test_decompress_matches_oracle(mode, G, d, kind):
    """d = 320, 576, 832: mode 2 with G = 32 / 64 takes two slices per nope lane
    ((d - 64) / 32 a multiple of 4); d = 128, 1024 and G = 16 one slice."""
    _same(_case(203, d, mode, G, kind, seed=31))


@pytest.mark.parametrize("G", [32, 64])
@pytest.mark.parametrize("T", [1, 15, 16, 17, 6037])
def test_decompress_mode2_block_tails(G, T):
    """Row counts around the 16-row blocks of the mode-2 chunk layout."""
    _same(_case(T, 576, 2, G, seed=47))


@pytest.mark.parametrize("mode,G", [(0, 64), (1, 64), (2, 32)])
@pytest.mark.parametrize("extra,pad", [(0, 0), (1, 0), (3, 40), (16, 1000)])
def test_decompress_row_alignments(mode, G, extra, pad):
    """headDim tails and block strides that make packed rows start at every alignment."""
    _same(_case(77, 320, mode, G, extra=extra, pad=pad, seed=33))


@pytest.mark.parametrize("y_extra,y_shift", [(0, 1), (8, 0), (3, 5)])
def test_decompress_strided_and_misaligned_y(y_extra, y_shift):
    _same(_case(61, 576, 0, seed=35), y_extra=y_extra, y_shift=y_shift)


@pytest.mark.parametrize("T", [0, 1, 7, 31, 33, 6037])
def test_decompress_ragged_counts(T):
    _same(_case(T, 576, 2, 32, seed=37))


def test_decompress_bad_slots_fault_and_int64():
    case = _case(64, 576, 0, seed=39, slot_dtype=np.int64)
    slots = case.arrays["slot_mapping"].copy()
    slots[3] = case.caches["cache"].num_slots
    slots[10] = -5
    y = _same(case, slots=slots)
    assert np.all(y[3] == MARK) and np.all(y[10] == MARK)


@pytest.mark.parametrize("name", ["compress_mode0_T262144_d576", "compress_mode2_G32_T262144_d576",
                                  "compress_mode1_T64_d256"])
def test_decompress_named_workloads_full_size(name):
    _same(W.CONFIGS[name]())


@pytest.mark.parametrize("kind", ["normal", "wide"])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("d", [128, 576, 1088])
def test_decompress_f16_rows(mode, d, kind):
    """Rows compressed from float16 x decode into float16 y (quantMode 0/1)."""
    _same(_case(203, d, mode, kind=kind, seed=41, x_dtype="f16"))


def test_decompress_f16_full_size():
    _same(W.CONFIGS["compress_mode0_f16_T262144_d576"]())
