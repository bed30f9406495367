"""CPU oracle of the per-token KV-cache epilogue -- TEST INFRASTRUCTURE.

This package states, in plain C (kvq_oracle.c) behind a thin numpy/ctypes
wrapper, what the four epilogue operations compute.  Only the tests, the
smoke check (``__graft_entry__.smoke``) and the benchmark's CPU-baseline leg
may import it.  The CUDA library never uses it and shares no code with it.

The token Compressor (aclnnCompressor, C128A form) is oracle/compressor.py:
numpy in float64, pinned by tests/test_oracle_compressor.py.

Pinned by tests/test_oracle_codecs.py and tests/test_oracle_ops.py.  Parity
unpinned (conventions with nothing on the pages to check against): the
packed-row segment order, the FP4 nibble order, the padding bytes, and the
indexer quant_mode numbers other than 0.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import build as _build

_LIB: Optional[ctypes.CDLL] = None

FMT_IDS = {"e4m3": 0, "e5m2": 1, "e2m1": 2, "bf16": 3, "f16": 4}
IN_DTYPES = {"bf16": 0, "f16": 1, "i32": 2, "f32": 3}
CACHE_DTYPES = {"bf16": 0, "f16": 1, "e4m3": 2, "e5m2": 3, "i8": 4}
RMS_CACHE_MODES = {"Norm": 0, "PA": 1, "PA_BNSD": 2, "PA_BLK_BNSD": 3}
FAULT_SLOT_RANGE = 0x1

_i64 = ctypes.c_int64
_vp = ctypes.c_void_p


class _Paged(ctypes.Structure):
    _fields_ = [("base", _vp), ("num_blocks", _i64), ("block_size", _i64),
                ("row_bytes", _i64), ("block_stride", _i64)]


class _CacheOut(ctypes.Structure):
    _fields_ = [("geom", _Paged), ("dtype", ctypes.c_int), ("scale", _vp), ("scale_n", _i64),
                ("offset", _vp), ("offset_n", _i64)]


class _DrqArgs(ctypes.Structure):
    _fields_ = [("x", _vp), ("x_dtype", ctypes.c_int), ("B", _i64), ("S", _i64), ("H", _i64),
                ("cos", _vp), ("sin", _vp), ("cos_dtype", ctypes.c_int),
                ("k_cache", _vp), ("v_cache", _vp), ("c0", _i64), ("c1", _i64),
                ("k_block_stride", _i64), ("v_block_stride", _i64),
                ("indices", _vp), ("scale_k", _vp), ("scale_v", _vp), ("offset_k", _vp),
                ("offset_v", _vp), ("weight_scale", _vp), ("activation_scale", _vp),
                ("bias", _vp), ("bias_dtype", ctypes.c_int), ("size_splits", _i64 * 3),
                ("D", _i64), ("cache_mode", ctypes.c_int), ("kv_output", ctypes.c_int),
                ("q_out", _vp), ("k_out", _vp), ("v_out", _vp)]


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.kvqo_kv_cache_col.restype = _i64
        L.kvqo_kv_cache_col.argtypes = [_i64, ctypes.c_int, _i64]
        L.kvqo_indexer_scale_col.restype = _i64
        L.kvqo_indexer_scale_col.argtypes = [_i64, ctypes.c_int]
        L.kvqo_encode_array.argtypes = [ctypes.c_int, _vp, _i64, ctypes.c_int, _vp]
        L.kvqo_decode_array.argtypes = [ctypes.c_int, _vp, _i64, _vp]
        L.kvqo_e8m0_ceil_array.argtypes = [_vp, _i64, _vp]
        L.kvqo_int8_static_array.argtypes = [_vp, _i64, _vp]
        L.kvqo_kv_compress_epilog.argtypes = [_vp, ctypes.c_int, _i64, _i64, _i64, _vp, ctypes.POINTER(_Paged),
                                              ctypes.c_int, _i64, ctypes.c_float, _vp]
        L.kvqo_indexer_quant_cache.argtypes = [_vp, ctypes.c_int, _i64, _i64, _i64, _vp,
                                               ctypes.POINTER(_Paged), ctypes.c_int,
                                               ctypes.POINTER(_Paged), ctypes.c_int, _vp]
        L.kvqo_kv_rmsnorm_rope_cache.argtypes = [_vp, ctypes.c_int, _i64, _i64, _i64, _i64, _vp, _vp,
                                                 _vp, _vp, ctypes.c_int, ctypes.POINTER(_CacheOut),
                                                 ctypes.POINTER(_CacheOut), ctypes.c_float, _vp]
        L.kvqo_dequant_rope_quant_kvcache.argtypes = [ctypes.POINTER(_DrqArgs), _vp]
        L.kvqo_kv_decompress.argtypes = [ctypes.POINTER(_Paged), _vp, _i64, _i64, ctypes.c_int, _i64,
                                         ctypes.c_float, ctypes.c_int, _vp, _i64, _vp]
        _LIB = L
    return _LIB


def _ptr(a: Optional[np.ndarray]) -> Optional[int]:
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what}: parameters it cannot compute (status {rc})")


# ----------------------------------------------------------------------------
# codecs
# ----------------------------------------------------------------------------
def encode(fmt: str, values, saturate: bool = True) -> np.ndarray:
    v = np.ascontiguousarray(values, dtype=np.float32).ravel()
    out = np.empty(v.size, dtype=np.uint32)
    _check(lib().kvqo_encode_array(FMT_IDS[fmt], _ptr(v), v.size, int(saturate), _ptr(out)), "encode")
    return out


def decode(fmt: str, codes) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint32).ravel()
    out = np.empty(c.size, dtype=np.float32)
    _check(lib().kvqo_decode_array(FMT_IDS[fmt], _ptr(c), c.size, _ptr(out)), "decode")
    return out


def e8m0_ceil(q) -> np.ndarray:
    v = np.ascontiguousarray(q, dtype=np.float32).ravel()
    out = np.empty(v.size, dtype=np.uint8)
    lib().kvqo_e8m0_ceil_array(_ptr(v), v.size, _ptr(out))
    return out


def int8_static(v) -> np.ndarray:
    a = np.ascontiguousarray(v, dtype=np.float32).ravel()
    out = np.empty(a.size, dtype=np.int8)
    lib().kvqo_int8_static_array(_ptr(a), a.size, _ptr(out))
    return out


def kv_cache_col(d: int, quant_mode: int, group_size: int = 64) -> int:
    return int(lib().kvqo_kv_cache_col(d, quant_mode, group_size))


def indexer_scale_col(d: int, quant_mode: int) -> int:
    return int(lib().kvqo_indexer_scale_col(d, quant_mode))


# ----------------------------------------------------------------------------
# paged caches: a byte buffer plus the geometry of a [blockNum, blockSize, 1,
# headDim] view into it (only the block dimension may be strided)
# ----------------------------------------------------------------------------
@dataclass
class Paged:
    storage: np.ndarray      # uint8, 1-D, writable; updated in place
    offset: int              # byte offset of block 0, row 0
    num_blocks: int
    block_size: int
    row_bytes: int           # bytes per slot row (headDim x element size)
    block_stride: int        # bytes between blocks

    def c(self) -> _Paged:
        assert self.storage.dtype == np.uint8 and self.storage.flags["C_CONTIGUOUS"]
        last = self.offset + (self.num_blocks - 1) * self.block_stride + self.block_size * self.row_bytes
        assert 0 <= self.offset and last <= self.storage.size, "geometry outside storage"
        return _Paged(self.storage.ctypes.data + self.offset, self.num_blocks, self.block_size,
                      self.row_bytes, self.block_stride)


def _slots(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a).ravel(), dtype=np.int64)


def _row_chunks(T: int, threads: int):
    n = max(1, min(threads, T))
    bounds = np.linspace(0, T, n + 1).astype(np.int64)
    return [(int(bounds[i]), int(bounds[i + 1])) for i in range(n) if bounds[i + 1] > bounds[i]]


def _parallel_rows(T: int, threads: int, fn) -> int:
    """Run fn(row_lo, row_hi) -> fault bits over row chunks.  Every row writes only
    its own slot row, so chunks are independent; ctypes releases the GIL."""
    chunks = _row_chunks(T, threads)
    if len(chunks) <= 1:
        return fn(0, T)
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(len(chunks)) as ex:
        bits = list(ex.map(lambda c: fn(*c), chunks))
    out = 0
    for b in bits:
        out |= b
    return out


def kv_compress_epilog(x_bits: np.ndarray, slot_mapping, cache: Paged, quant_mode: int,
                       quant_group_size: int = 64, x_scale: float = 1.0, threads: int = 1,
                       x_dtype: str = "bf16") -> int:
    """x_bits: uint16 bit patterns [..., d] of bf16 (or, in quantMode 0/1, f16) values.
    Updates cache.storage; returns fault bits."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    d = x.shape[-1]
    T = x.size // d
    x = x.reshape(T, d)
    s = _slots(slot_mapping)
    assert s.size == T
    pc = cache.c()

    def run(lo, hi):
        faults = np.zeros(1, dtype=np.uint32)
        rc = lib().kvqo_kv_compress_epilog(x[lo:].ctypes.data, IN_DTYPES[x_dtype], hi - lo, d, d, s[lo:].ctypes.data,
                                           ctypes.byref(pc), quant_mode, quant_group_size,
                                           ctypes.c_float(x_scale), _ptr(faults))
        _check(rc, "kv_compress_epilog")
        return int(faults[0])
    return _parallel_rows(T, threads, run)


def kv_decompress(cache: Paged, slot_mapping, d: int, quant_mode: int, quant_group_size: int = 64,
                  x_scale: float = 1.0, y: Optional[np.ndarray] = None, threads: int = 1, y_dtype: str = "bf16"):
    """Decode the packed rows named by slot_mapping into bit patterns y [T, d] of bf16
    (or f16 in quantMode 0/1: the dtype of the compressed x) values; rows of skipped
    tokens keep y's initial contents, zeros by default.  Returns (y, fault bits)."""
    s = _slots(slot_mapping)
    T = s.size
    if y is None:
        y = np.zeros((T, d), dtype=np.uint16)
    assert y.dtype == np.uint16 and y.shape == (T, d) and y.flags["C_CONTIGUOUS"]
    pc = cache.c()

    def run(lo, hi):
        faults = np.zeros(1, dtype=np.uint32)
        rc = lib().kvqo_kv_decompress(ctypes.byref(pc), s[lo:].ctypes.data, hi - lo, d, quant_mode,
                                      quant_group_size, ctypes.c_float(x_scale), IN_DTYPES[y_dtype],
                                      y[lo:].ctypes.data, d,
                                      _ptr(faults))
        _check(rc, "kv_decompress")
        return int(faults[0])
    return y, _parallel_rows(T, threads, run)


def indexer_quant_cache(x_bits: np.ndarray, x_dtype: str, slot_mapping, cache: Paged, cache_fp8: str,
                        cache_scale: Paged, quant_mode: int, threads: int = 1) -> int:
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    d = x.shape[-1]
    T = x.size // d
    x = x.reshape(T, d)
    s = _slots(slot_mapping)
    assert s.size == T
    pc, ps = cache.c(), cache_scale.c()

    def run(lo, hi):
        faults = np.zeros(1, dtype=np.uint32)
        rc = lib().kvqo_indexer_quant_cache(x[lo:].ctypes.data, IN_DTYPES[x_dtype], hi - lo, d, d,
                                            s[lo:].ctypes.data, ctypes.byref(pc),
                                            1 if cache_fp8 == "e5m2" else 0, ctypes.byref(ps), quant_mode,
                                            _ptr(faults))
        _check(rc, "indexer_quant_cache")
        return int(faults[0])
    return _parallel_rows(T, threads, run)


@dataclass
class CacheOut:
    paged: Paged
    dtype: str                          # bf16 | f16 | e4m3 | e5m2 | i8
    scale: Optional[np.ndarray] = None  # float32, 1 value or one per channel
    offset: Optional[np.ndarray] = None


def _cache_out(co: CacheOut, keep: list) -> _CacheOut:
    sc = None if co.scale is None else np.ascontiguousarray(co.scale, dtype=np.float32).ravel()
    of = None if co.offset is None else np.ascontiguousarray(co.offset, dtype=np.float32).ravel()
    keep += [sc, of]
    return _CacheOut(co.paged.c(), CACHE_DTYPES[co.dtype], _ptr(sc), 0 if sc is None else sc.size,
                     _ptr(of), 0 if of is None else of.size)


def kv_rmsnorm_rope_cache(kv_bits: np.ndarray, kv_dtype: str, Dv: int, gamma_bits, cos_bits, sin_bits,
                          index, cache_mode: str, k_cache: CacheOut, ckv_cache: CacheOut,
                          epsilon: float) -> int:
    """kv_bits: uint16 [B, 1, S, D]; cos/sin [B, 1, S, Dk]; gamma [Dv]."""
    kv = np.ascontiguousarray(kv_bits, dtype=np.uint16)
    B, N, S, D = kv.shape
    assert N == 1
    g = np.ascontiguousarray(gamma_bits, dtype=np.uint16)
    c = np.ascontiguousarray(cos_bits, dtype=np.uint16)
    s = np.ascontiguousarray(sin_bits, dtype=np.uint16)
    idx = _slots(index)
    keep: list = []
    ko, co = _cache_out(k_cache, keep), _cache_out(ckv_cache, keep)
    faults = np.zeros(1, dtype=np.uint32)
    rc = lib().kvqo_kv_rmsnorm_rope_cache(_ptr(kv), IN_DTYPES[kv_dtype], B, S, D, Dv, _ptr(g), _ptr(c),
                                          _ptr(s), _ptr(idx), RMS_CACHE_MODES[cache_mode],
                                          ctypes.byref(ko), ctypes.byref(co), ctypes.c_float(epsilon),
                                          _ptr(faults))
    _check(rc, "kv_rmsnorm_rope_cache")
    return int(faults[0])


def dequant_rope_quant_kvcache(x: np.ndarray, x_dtype: str, cos_bits, sin_bits, cos_dtype: str,
                               k_cache: Paged, v_cache: Paged, indices, scale_k, scale_v,
                               offset_k=None, offset_v=None, weight_scale=None, activation_scale=None,
                               bias=None, bias_dtype: str = "f32", size_splits=(0, 0, 0),
                               cache_mode: str = "contiguous", kv_output: bool = False):
    """x: [B, S, H] or [B, H] (int32 values, or uint16 bit patterns for bf16/f16).

    k_cache / v_cache: int8 caches [c0, c1, Nkv, D] as Paged with num_blocks = c0,
    block_size = c1 and row_bytes = Nkv * D.  Returns (q_out, k_out, v_out, faults);
    the 16-bit outputs are uint16 bit patterns of the cos dtype.
    """
    if x.ndim == 2:
        B, H = x.shape
        S = 1
    else:
        B, S, H = x.shape
    xa = np.ascontiguousarray(x, dtype=np.int32 if x_dtype == "i32" else np.uint16)
    # D is the head dimension (the caches' last dimension and cos/sin's last
    # dimension); a cache row holds the Nkv * D int8 values of one token.
    assert k_cache.row_bytes == size_splits[1] and v_cache.row_bytes == size_splits[2]
    D = int(np.asarray(cos_bits).shape[-1])
    Nq, Nkv = size_splits[0] // D, size_splits[1] // D
    q_out = np.zeros((B, S, Nq, D), dtype=np.uint16)
    k_out = np.zeros((B, S, Nkv, D), dtype=np.uint16) if kv_output else None
    v_out = np.zeros((B, S, Nkv, D), dtype=np.uint16) if kv_output else None
    keep = []

    def f32(a):
        if a is None:
            return None
        r = np.ascontiguousarray(a, dtype=np.float32).ravel()
        keep.append(r)
        return r

    c = np.ascontiguousarray(cos_bits, dtype=np.uint16)
    s = np.ascontiguousarray(sin_bits, dtype=np.uint16)
    idx = _slots(indices)
    if bias is not None:
        bdt = {"f32": np.float32, "f16": np.uint16, "bf16": np.uint16, "i32": np.int32}[bias_dtype]
        bias_arr = np.ascontiguousarray(bias, dtype=bdt).ravel()
    else:
        bias_arr = None
    sk, sv, ok, ov, ws, act = (f32(scale_k), f32(scale_v), f32(offset_k), f32(offset_v),
                               f32(weight_scale), f32(activation_scale))
    assert k_cache.storage.flags["C_CONTIGUOUS"] and v_cache.storage.flags["C_CONTIGUOUS"]
    args = _DrqArgs()
    args.x, args.x_dtype, args.B, args.S, args.H = _ptr(xa), IN_DTYPES[x_dtype], B, S, H
    args.cos, args.sin, args.cos_dtype = _ptr(c), _ptr(s), IN_DTYPES[cos_dtype]
    kc, vc = k_cache.c(), v_cache.c()
    args.k_cache, args.v_cache = kc.base, vc.base
    args.c0, args.c1 = k_cache.num_blocks, k_cache.block_size
    args.k_block_stride, args.v_block_stride = k_cache.block_stride, v_cache.block_stride
    args.indices = _ptr(idx)
    args.scale_k, args.scale_v, args.offset_k, args.offset_v = _ptr(sk), _ptr(sv), _ptr(ok), _ptr(ov)
    args.weight_scale, args.activation_scale = _ptr(ws), _ptr(act)
    args.bias = _ptr(bias_arr)
    args.bias_dtype = IN_DTYPES[bias_dtype]
    args.size_splits = (_i64 * 3)(*size_splits)
    args.D = D
    args.cache_mode = 1 if cache_mode == "page" else 0
    args.kv_output = int(kv_output)
    args.q_out, args.k_out, args.v_out = _ptr(q_out), _ptr(k_out), _ptr(v_out)
    faults = np.zeros(1, dtype=np.uint32)
    _check(lib().kvqo_dequant_rope_quant_kvcache(ctypes.byref(args), _ptr(faults)), "dequant_rope_quant_kvcache")
    if x.ndim == 2:
        q_out = q_out.reshape(B, Nq, D)
        if kv_output:
            k_out, v_out = k_out.reshape(B, Nkv, D), v_out.reshape(B, Nkv, D)
    return q_out, k_out, v_out, int(faults[0])
