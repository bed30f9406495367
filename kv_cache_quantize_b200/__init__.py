"""B200-native per-token KV-cache epilogue: Python binding of libkvq.so.

Thin ctypes marshalling over the C ABI in include/kvq.h -- every step of the
epilogue runs in the library's sm_100a kernels; torch supplies device memory
and streams only.  There is no fallback: if the CUDA library is missing, the
first call raises.

Operations (same names as the C ABI without the ``kvq_`` prefix):
  kv_compress_epilog, indexer_quant_cache, kv_rmsnorm_rope_cache,
  dequant_rope_quant_kvcache; the packed-row decoder kv_decompress;
  utilities get_error, kv_cache_col, indexer_scale_col, convert.

Device faults.  A call returns once its kernel is enqueued; a slot outside
the cache (other than -1), or a pipeline wait that gave up, is not an error of
the call but a bit in the device's fault word.  Call ``get_error()`` to read
and clear those bits, or pass ``check=True`` to an operation, which waits for
the stream and raises ``KvqFault`` if any bit is set.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

__all__ = [
    "KvqError", "KvqFault", "lib", "library_path", "kv_compress_epilog", "kv_decompress", "indexer_quant_cache",
    "kv_rmsnorm_rope_cache",
    "dequant_rope_quant_kvcache", "compressor", "get_error", "kv_cache_col", "indexer_scale_col", "convert", "selftest", "scatter_rows",
    "FAULT_SLOT_RANGE", "FAULT_TIMEOUT", "STATUS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libkvq.so")
_LIB: Optional[ctypes.CDLL] = None

MAX_DIMS = 8
FAULT_SLOT_RANGE = 0x1
FAULT_TIMEOUT = 0x2
STATUS = {0: "KVQ_OK", 1: "KVQ_ERR_NULL", 2: "KVQ_ERR_NDIM", 3: "KVQ_ERR_SHAPE", 4: "KVQ_ERR_DTYPE",
          5: "KVQ_ERR_ATTR", 6: "KVQ_ERR_LAYOUT", 7: "KVQ_ERR_CAPACITY", 8: "KVQ_ERR_CUDA",
          9: "KVQ_ERR_UNSUPPORTED"}

_DTYPES = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2, torch.int32: 3, torch.int64: 4,
           torch.int8: 5, torch.uint8: 6, torch.float8_e4m3fn: 7, torch.float8_e5m2: 8,
           torch.float8_e8m0fnu: 9}

RMS_CACHE_MODES = {"Norm": 0, "PA": 1, "PA_BNSD": 2, "PA_BLK_BNSD": 3, "PA_NZ": 4, "PA_BLK_NZ": 5}
DRQ_CACHE_MODES = {"contiguous": 0, "page": 1}
INDEXER_MODES = {"mxfp8": 0, "fp8": 1, "hifloat8": 2, "mxfp4": 3}
CONVERT_FORMATS = {"e4m3": 0, "e5m2": 1, "e2m1": 2, "bf16": 3, "e8m0": 4, "i8": 5}


class KvqTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * MAX_DIMS), ("stride", ctypes.c_int64 * MAX_DIMS)]


class KvqError(RuntimeError):
    def __init__(self, op: str, status: int):
        self.status = status
        super().__init__(f"{op}: {STATUS.get(status, status)} ({lib().kvq_status_string(status).decode()})")


class KvqFault(RuntimeError):
    """Device fault bits (FAULT_SLOT_RANGE, FAULT_TIMEOUT) found after an operation run with check=True."""
    def __init__(self, op: str, bits: int):
        self.bits = bits
        names = [n for b, n in ((FAULT_SLOT_RANGE, "FAULT_SLOT_RANGE"), (FAULT_TIMEOUT, "FAULT_TIMEOUT")) if bits & b]
        super().__init__(f"{op}: device fault bits {bits:#x} ({', '.join(names) or 'unknown'})")


_P = ctypes.POINTER(KvqTensor)


def lib() -> ctypes.CDLL:
    """Load libkvq.so (built by kv_cache_quantize_b200/build.py); raise if it is missing."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(library_path):
            raise RuntimeError(f"CUDA library not built: {library_path} is missing "
                               "(run `python -c 'import __graft_entry__ as g; g.build()'`)")
        L = ctypes.CDLL(library_path)
        i32, i64, vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
        L.kvq_kv_compress_epilog.argtypes = [_P, _P, _P, i32, i32, ctypes.c_float, vp]
        L.kvq_kv_decompress.argtypes = [_P, _P, _P, i32, i32, ctypes.c_float, vp]
        L.kvq_indexer_quant_cache.argtypes = [_P, _P, _P, _P, i32, vp]
        L.kvq_kv_rmsnorm_rope_cache.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_float, i32, vp]
        L.kvq_dequant_rope_quant_kvcache.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                                     ctypes.POINTER(i64), i32, i32, i32, i32, i32, _P, _P, _P, vp]
        L.kvq_get_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        L.kvq_scatter_rows.argtypes = [_P, _P, _P, i64, vp]
        L.kvq_compressor.argtypes = [_P, _P, _P, _P, _P, i32, vp]
        L.kvq_convert.argtypes = [i32, vp, i64, vp, vp]
        L.kvq_selftest.argtypes = [i32, ctypes.POINTER(ctypes.c_uint64), vp]
        L.kvq_kv_cache_col.argtypes = [i64, i32, i32]
        L.kvq_kv_cache_col.restype = i64
        L.kvq_indexer_scale_col.argtypes = [i64, i32]
        L.kvq_indexer_scale_col.restype = i64
        L.kvq_status_string.argtypes = [i32]
        L.kvq_status_string.restype = ctypes.c_char_p
        L.kvq_version.restype = i32
        for name in ("kvq_kv_compress_epilog", "kvq_kv_decompress", "kvq_indexer_quant_cache",
                     "kvq_kv_rmsnorm_rope_cache",
                     "kvq_dequant_rope_quant_kvcache", "kvq_get_error", "kvq_convert", "kvq_selftest",
                     "kvq_scatter_rows", "kvq_compressor"):
            getattr(L, name).restype = i32
        _LIB = L
    return _LIB


def desc(t: Optional[torch.Tensor]) -> Optional[KvqTensor]:
    """Describe a tensor for the C ABI (device pointer, dtype, shape, strides in elements)."""
    if t is None:
        return None
    if t.dtype not in _DTYPES:
        raise TypeError(f"dtype {t.dtype} has no kvq equivalent")
    if t.dim() > MAX_DIMS:
        raise ValueError("too many dimensions")
    d = KvqTensor()
    d.data = t.data_ptr() if t.numel() > 0 else 0
    d.dtype = _DTYPES[t.dtype]
    d.ndim = t.dim()
    for i, (s, st) in enumerate(zip(t.shape, t.stride())):
        d.shape[i] = s
        d.stride[i] = st
    return d


def _ref(d: Optional[KvqTensor]):
    return None if d is None else ctypes.byref(d)


def _one_device(op: str, *tensors) -> Optional[torch.device]:
    """Every non-empty tensor of a call must live on one CUDA device: the kernels
    dereference the pointers on the device, and a host pointer or another
    device's memory would fault there instead of failing here.  Returns that
    device (None when every tensor is empty)."""
    dev = None
    for t in tensors:
        if t is None or t.numel() == 0:
            continue
        if not t.is_cuda:
            raise ValueError(f"{op}: tensors must be on a CUDA device, got one on {t.device}")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{op}: tensors on {dev} and {t.device}; all must be on one device")
    return dev


def _on(dev: Optional[torch.device]):
    """Make the call's device current while the library runs: it sizes grids,
    sets kernel attributes and launches on the current device."""
    if dev is None or dev.index is None or dev.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(dev)


def _stream(stream, *tensors) -> int:
    if stream is None:
        dev = next((t.device for t in tensors if t is not None and t.is_cuda), None)
        if dev is None:
            return 0
        return torch.cuda.current_stream(dev).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(op: str, status: int) -> None:
    if status != 0:
        raise KvqError(op, status)


def _faults(op: str, check: bool, stream: int) -> None:
    """With check=True: wait for the stream, read and clear the fault word, raise if set."""
    if not check:
        return
    bits = ctypes.c_uint32(0)
    _check(op, lib().kvq_get_error(stream, ctypes.byref(bits)))
    if bits.value:
        raise KvqFault(op, int(bits.value))


# ---------------------------------------------------------------------------
def kv_compress_epilog(x: torch.Tensor, slot_mapping: torch.Tensor, cache: torch.Tensor, quant_mode: int,
                       quant_group_size: int = 64, x_scale: float = 1.0, stream=None, check: bool = False) -> None:
    """In-place group quantisation of x's rows into the paged cache (see kvq_kv_compress_epilog).
    Device faults (a bad slot) are reported by get_error(), or raised here with check=True."""
    with _on(_one_device("kv_compress_epilog", x, slot_mapping, cache)):
        st = _stream(stream, x)
        _check("kv_compress_epilog", lib().kvq_kv_compress_epilog(
            _ref(desc(x)), _ref(desc(slot_mapping)), _ref(desc(cache)), int(quant_mode), int(quant_group_size),
            float(x_scale), st))
        _faults("kv_compress_epilog", check, st)


def kv_decompress(cache: torch.Tensor, slot_mapping: torch.Tensor, y: torch.Tensor, quant_mode: int,
                  quant_group_size: int = 64, x_scale: float = 1.0, stream=None, check: bool = False) -> torch.Tensor:
    """Decode the packed rows named by slot_mapping into the bf16 rows of y (see kvq_kv_decompress);
    rows whose slot is -1 keep their contents.  Returns y.  Device faults (a bad slot) are
    reported by get_error(), or raised here with check=True."""
    with _on(_one_device("kv_decompress", cache, slot_mapping, y)):
        st = _stream(stream, y)
        _check("kv_decompress", lib().kvq_kv_decompress(
            _ref(desc(cache)), _ref(desc(slot_mapping)), _ref(desc(y)), int(quant_mode), int(quant_group_size),
            float(x_scale), st))
        _faults("kv_decompress", check, st)
    return y


def indexer_quant_cache(x: torch.Tensor, cache: torch.Tensor, cache_scale: torch.Tensor,
                        slot_mapping: torch.Tensor, quant_mode="mxfp8", stream=None, check: bool = False) -> None:
    """In-place mxfp8 / fp8 / mxfp4 quantisation into cache and cache_scale (see kvq_indexer_quant_cache).
    Device faults (a bad slot) are reported by get_error(), or raised here with check=True."""
    mode = INDEXER_MODES[quant_mode] if isinstance(quant_mode, str) else int(quant_mode)
    with _on(_one_device("indexer_quant_cache", x, cache, cache_scale, slot_mapping)):
        st = _stream(stream, x)
        _check("indexer_quant_cache", lib().kvq_indexer_quant_cache(
            _ref(desc(x)), _ref(desc(cache)), _ref(desc(cache_scale)), _ref(desc(slot_mapping)), mode, st))
        _faults("indexer_quant_cache", check, st)


def kv_rmsnorm_rope_cache(kv: torch.Tensor, gamma: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor,
                          index: torch.Tensor, k_cache: torch.Tensor, ckv_cache: torch.Tensor,
                          k_scale: Optional[torch.Tensor] = None, ckv_scale: Optional[torch.Tensor] = None,
                          k_offset: Optional[torch.Tensor] = None, ckv_offset: Optional[torch.Tensor] = None,
                          epsilon: float = 1e-5, cache_mode="PA_BNSD", stream=None, check: bool = False) -> None:
    """RMSNorm of kv[..., :Dv] -> ckv_cache and interleaved RoPE of kv[..., Dv:] -> k_cache, in place.
    Device faults (a bad index) are reported by get_error(), or raised here with check=True."""
    mode = RMS_CACHE_MODES[cache_mode] if isinstance(cache_mode, str) else int(cache_mode)
    with _on(_one_device("kv_rmsnorm_rope_cache", kv, gamma, cos, sin, index, k_cache, ckv_cache, k_scale,
                         ckv_scale, k_offset, ckv_offset)):
        st = _stream(stream, kv)
        _check("kv_rmsnorm_rope_cache", lib().kvq_kv_rmsnorm_rope_cache(
            _ref(desc(kv)), _ref(desc(gamma)), _ref(desc(cos)), _ref(desc(sin)), _ref(desc(index)),
            _ref(desc(k_cache)), _ref(desc(ckv_cache)), _ref(desc(k_scale)), _ref(desc(ckv_scale)),
            _ref(desc(k_offset)), _ref(desc(ckv_offset)), float(epsilon), mode, st))
        _faults("kv_rmsnorm_rope_cache", check, st)


def dequant_rope_quant_kvcache(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor, k_cache: torch.Tensor,
                               v_cache: torch.Tensor, indices: torch.Tensor, scale_k: torch.Tensor,
                               scale_v: torch.Tensor, offset_k: Optional[torch.Tensor] = None,
                               offset_v: Optional[torch.Tensor] = None,
                               weight_scale: Optional[torch.Tensor] = None,
                               activation_scale: Optional[torch.Tensor] = None,
                               bias: Optional[torch.Tensor] = None, size_splits: Sequence[int] = (),
                               quant_mode: str = "static", layout: str = "BSND", kv_output: bool = False,
                               cache_mode: str = "contiguous", q_out: Optional[torch.Tensor] = None,
                               k_out: Optional[torch.Tensor] = None, v_out: Optional[torch.Tensor] = None,
                               stream=None, check: bool = False) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Fused int32 dequant -> q/k/v split -> half-rotation RoPE -> static int8 quant -> cache write.

    Returns (q_out, k_out, v_out); output tensors not supplied are allocated with
    the shapes of the page's shape inference ([B,S,N,D] for a 3-D x, [B,N,D] for a
    2-D x; k_out / v_out with a zero first dimension when kv_output is false).
    Device faults (a bad index) are reported by get_error(), or raised here with check=True.
    """
    D = k_cache.shape[-1]
    splits = list(size_splits)
    Nq = splits[0] // D if splits and D else 0
    Nkv = splits[1] // D if len(splits) > 1 and D else 0
    lead = tuple(x.shape[:-1])
    odt = cos.dtype
    if q_out is None:
        q_out = torch.empty(lead + (Nq, D), dtype=odt, device=x.device)
    if k_out is None:
        k_out = torch.empty(lead + (Nkv, D) if kv_output else (0,) + lead[1:] + (Nkv, D), dtype=odt,
                            device=x.device)
    if v_out is None:
        v_out = torch.empty(lead + (Nkv, D) if kv_output else (0,) + lead[1:] + (Nkv, D), dtype=odt,
                            device=x.device)
    dev = _one_device("dequant_rope_quant_kvcache", x, cos, sin, k_cache, v_cache, indices, scale_k, scale_v,
                      offset_k, offset_v, weight_scale, activation_scale, bias, q_out, k_out, v_out)
    arr = (ctypes.c_int64 * max(1, len(splits)))(*splits)
    qm = {"static": 0}.get(quant_mode, -1) if isinstance(quant_mode, str) else int(quant_mode)
    lo = {"BSND": 0}.get(layout, -1) if isinstance(layout, str) else int(layout)
    cm = DRQ_CACHE_MODES.get(cache_mode, -1) if isinstance(cache_mode, str) else int(cache_mode)
    with _on(dev):
        st = _stream(stream, x)
        _check("dequant_rope_quant_kvcache", lib().kvq_dequant_rope_quant_kvcache(
            _ref(desc(x)), _ref(desc(cos)), _ref(desc(sin)), _ref(desc(k_cache)), _ref(desc(v_cache)),
            _ref(desc(indices)), _ref(desc(scale_k)), _ref(desc(scale_v)), _ref(desc(offset_k)),
            _ref(desc(offset_v)), _ref(desc(weight_scale)), _ref(desc(activation_scale)), _ref(desc(bias)),
            arr, len(splits), qm, lo, int(bool(kv_output)), cm, _ref(desc(q_out)),
            _ref(desc(k_out)) if kv_output else None, _ref(desc(v_out)) if kv_output else None, st))
        _faults("dequant_rope_quant_kvcache", check, st)
    return q_out, k_out, v_out


def compressor(x: torch.Tensor, w_kv: torch.Tensor, w_gate: torch.Tensor, ape: torch.Tensor,
               cmp_kv: Optional[torch.Tensor] = None, cmp_ratio: int = 128, stream=None,
               check: bool = False) -> torch.Tensor:
    """The token Compressor (see kvq_compressor): C128A form with w_kv [D, H] -- per group of
    cmp_ratio token rows and channel, the softmax over the group of (x @ w_gate^T + ape)
    weights x @ w_kv^T -- or C4A / C4Li form with w_kv [2D, H] and cmp_ratio 4 (a group's own
    four tokens through the first D weight rows, the next four through the last D).
    Returns cmp_kv [T / cmp_ratio, D] (allocated when not given: D is w_kv's rows when they
    are 128 or 512, else half of them)."""
    if cmp_kv is None:
        T = x.numel() // x.shape[-1] if x.dim() else 0
        rows = w_kv.shape[0]
        D = rows if rows in (128, 512) else rows // 2
        cmp_kv = torch.empty((T // max(1, int(cmp_ratio)), D), dtype=torch.bfloat16, device=x.device)
    with _on(_one_device("compressor", x, w_kv, w_gate, ape, cmp_kv)):
        st = _stream(stream, x)
        _check("compressor", lib().kvq_compressor(_ref(desc(x)), _ref(desc(w_kv)), _ref(desc(w_gate)),
                                                  _ref(desc(ape)), _ref(desc(cmp_kv)), int(cmp_ratio), st))
        _faults("compressor", check, st)
    return cmp_kv


def scatter_rows(x: torch.Tensor, slot_mapping: torch.Tensor, cache: torch.Tensor, out_bytes: int,
                 stream=None) -> None:
    """The compress kernels' memory access pattern without their arithmetic (see kvq_scatter_rows):
    each valid token's whole x row is read and its first out_bytes bytes land in its slot row."""
    with _on(_one_device("scatter_rows", x, slot_mapping, cache)):
        _check("scatter_rows", lib().kvq_scatter_rows(_ref(desc(x)), _ref(desc(slot_mapping)), _ref(desc(cache)),
                                                      int(out_bytes), _stream(stream, x)))


# ---------------------------------------------------------------------------
def get_error(stream=None, device=None) -> int:
    """Wait for the stream, return and clear the fault bits (FAULT_SLOT_RANGE, FAULT_TIMEOUT) of the
    device in one atomic read-and-clear on the device.  The device is `device`, else the
    stream's, else the current one."""
    if device is None and isinstance(stream, torch.cuda.Stream):
        device = stream.device
    dev = torch.device("cuda", torch.cuda._utils._get_device_index(device, optional=True))
    with _on(dev):
        if stream is None:
            stream = torch.cuda.current_stream(dev)
        bits = ctypes.c_uint32(0)
        _check("get_error", lib().kvq_get_error(_stream(stream), ctypes.byref(bits)))
    return int(bits.value)


def kv_cache_col(d: int, quant_mode: int, quant_group_size: int = 64) -> int:
    return int(lib().kvq_kv_cache_col(d, quant_mode, quant_group_size))


def indexer_scale_col(d: int, quant_mode) -> int:
    mode = INDEXER_MODES[quant_mode] if isinstance(quant_mode, str) else int(quant_mode)
    return int(lib().kvq_indexer_scale_col(d, mode))


def selftest(which: int, stream=None, device=None) -> int:
    """Run a device self-test of the kernels' arithmetic shortcuts; returns the mismatch count."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    out = ctypes.c_uint64(0)
    _check("selftest", lib().kvq_selftest(int(which), ctypes.byref(out), _stream(stream)))
    return int(out.value)


def convert(fmt: str, values: torch.Tensor, stream=None) -> torch.Tensor:
    """Encode a CUDA float32 tensor with the device codecs (one code per byte; bf16 -> int16 bits)."""
    if values.dtype != torch.float32 or not values.is_cuda or not values.is_contiguous():
        raise ValueError("convert needs a contiguous CUDA float32 tensor")
    f = CONVERT_FORMATS[fmt]
    out = torch.empty(values.shape, dtype=torch.int16 if fmt == "bf16" else torch.uint8, device=values.device)
    _check("convert", lib().kvq_convert(f, values.data_ptr(), values.numel(), out.data_ptr(),
                                        _stream(stream, values)))
    return out
