"""The C ABI without a GPU: the library loads, exports every symbol include/kvq.h
declares, and rejects bad arguments on the host.

Validation calls use descriptors whose data pointers are NULL: every rejection
happens before the data pointers are looked at, and a descriptor set that passes
validation stops at KVQ_ERR_NULL -- no call here can reach a kernel launch.
"""
import ctypes
import os
import re

import pytest
import torch

import kv_cache_quantize_b200 as kvq
import oracle
from _golden import read_table

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")

OK, ENULL, ENDIM, ESHAPE, EDTYPE, EATTR, ELAYOUT, ECAP, ECUDA, EUNSUP = range(10)


@pytest.fixture(scope="module")
def L():
    from kv_cache_quantize_b200 import build
    build.build()
    return kvq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_four_operations():
    names = declared_functions()
    for op in ("kvq_kv_compress_epilog", "kvq_kv_rmsnorm_rope_cache", "kvq_indexer_quant_cache",
               "kvq_dequant_rope_quant_kvcache"):
        assert op in names


def test_library_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), f"{n} declared in kvq.h but not exported"
    # and nothing else of the implementation leaks out of the shared object
    out = os.popen(f"nm -D --defined-only {kvq.library_path}").read()
    exported = sorted(set(re.findall(r" T (kvq_[a-z0-9_]+)$", out, flags=re.M)))
    assert exported == names


def test_sizes_match_golden_and_oracle(L):
    for r in read_table("layout_sizes.txt"):
        op, d, mode, g, expected = r[0], int(r[1]), int(r[2]), r[3], int(r[4])
        if op == "compress":
            assert kvq.kv_cache_col(d, mode, int(g)) == expected
        else:
            assert kvq.indexer_scale_col(d, mode) == expected
    for d in range(128, 8193, 64):
        for mode, G in ((0, 64), (1, 64), (2, 16), (2, 32), (2, 64)):
            if mode == 2 and (d - 64) % G:
                assert kvq.kv_cache_col(d, mode, G) == -1
                continue
            assert kvq.kv_cache_col(d, mode, G) == oracle.kv_cache_col(d, mode, G)
    assert kvq.kv_cache_col(64, 0, 64) == -1 and kvq.kv_cache_col(8256, 0, 64) == -1
    assert kvq.kv_cache_col(576, 3, 64) == -1 and kvq.kv_cache_col(576, 2, 48) == -1


def test_status_strings_and_version(L):
    for s in range(10):
        assert isinstance(L.kvq_status_string(s), bytes)
    assert L.kvq_version() >= 100


# ---------------------------------------------------------------------------
# host validation (NULL data pointers: never launches)
# ---------------------------------------------------------------------------
def D(shape, dtype, stride=None):
    t = kvq.KvqTensor()
    t.data = None
    t.dtype = {"bf16": 0, "f16": 1, "f32": 2, "i32": 3, "i64": 4, "i8": 5, "u8": 6, "e4m3": 7, "e5m2": 8,
               "e8m0": 9}[dtype]
    t.ndim = len(shape)
    if stride is None:
        stride, acc = [], 1
        for s in reversed(shape):
            stride.insert(0, acc)
            acc *= s
    for i, (s, st) in enumerate(zip(shape, stride)):
        t.shape[i], t.stride[i] = s, st
    return t


R = ctypes.byref


def ce(L, x, s, c, mode=0, G=64):
    return L.kvq_kv_compress_epilog(R(x), R(s), R(c), mode, G, ctypes.c_float(1.0), None)


def test_compress_validation(L):
    x, s, c = D([64, 576], "bf16"), D([64], "i32"), D([8, 16, 1, 672], "u8")
    assert ce(L, x, s, c) == ENULL                        # valid up to the (absent) data
    assert L.kvq_kv_compress_epilog(None, R(s), R(c), 0, 64, ctypes.c_float(1), None) == ENULL
    assert ce(L, D([64, 576], "f16"), s, c) == ENULL      # float16 x in quantMode 0 (and 1)
    assert ce(L, D([64, 576], "f16"), s, D([8, 16, 1, 648], "u8"), mode=1) == ENULL
    assert ce(L, D([64, 576], "f16"), s, D([8, 16, 1, 352], "u8"), mode=2, G=32) == EDTYPE   # mode 2: bf16 only
    assert ce(L, D([64, 576], "f32"), s, c) == EDTYPE
    assert ce(L, D([64, 600], "bf16"), s, c) == ESHAPE    # d % 64
    assert ce(L, D([64, 64], "bf16"), s, c) == ESHAPE     # d > 64
    assert ce(L, D([64, 8256], "bf16"), s, c) == ESHAPE   # d <= 8192
    assert ce(L, x, D([63], "i32"), c) == ESHAPE
    assert ce(L, x, D([64], "f32"), c) == EDTYPE
    assert ce(L, x, D([64, 2], "i32", [1, 64]), c) == ESHAPE
    assert ce(L, x, s, c, mode=3) == EATTR
    assert ce(L, x, s, D([8, 16, 1, 1024], "u8"), mode=2, G=48) == EATTR
    assert ce(L, D([64, 192], "bf16"), s, D([8, 16, 1, 1024], "u8"), mode=2, G=64) == ENULL
    assert ce(L, x, s, D([8, 16, 1, 671], "u8")) == ECAP  # headDim < kvCacheCol (672)
    assert ce(L, D([64, 256], "bf16"), s, D([8, 16, 1, 322], "u8"), mode=1) == ECAP   # 323 needed
    assert ce(L, D([64, 256], "bf16"), s, D([8, 16, 1, 323], "u8"), mode=1) == ENULL
    assert ce(L, x, s, D([8, 16, 2, 672], "u8")) == ESHAPE   # second-to-last dim must be 1
    assert ce(L, x, s, D([8, 16, 672], "u8")) == ENDIM
    assert ce(L, x, s, D([8, 16, 1, 672], "u8", [10752, 1344, 672, 1])) == ELAYOUT  # rows not contiguous
    assert ce(L, x, s, D([8, 16, 1, 672], "u8", [20000, 672, 672, 1])) == ENULL     # strided blocks are fine
    assert ce(L, x, s, D([8, 16, 1, 672], "u8", [5000, 672, 672, 1])) == ELAYOUT    # blocks overlap
    assert ce(L, D([64, 576], "bf16", [1, 64]), s, c) == ELAYOUT                     # column-major x
    assert ce(L, x, s, D([8, 16, 1, 672], "e4m3")) == EDTYPE
    assert ce(L, D([0, 576], "bf16"), D([0], "i32"), c) == OK                       # nothing to do


def kd(L, c, s, y, mode=0, G=64):
    return L.kvq_kv_decompress(R(c), R(s), R(y), mode, G, ctypes.c_float(1.0), None)


def test_decompress_validation(L):
    y, s, c = D([64, 576], "bf16"), D([64], "i32"), D([8, 16, 1, 672], "u8")
    assert kd(L, c, s, y) == ENULL                        # valid up to the (absent) data
    assert L.kvq_kv_decompress(R(c), R(s), None, 0, 64, ctypes.c_float(1), None) == ENULL
    assert kd(L, c, s, D([64, 576], "f16")) == ENULL      # float16 y for rows of float16 x (mode 0/1)
    assert kd(L, D([8, 16, 1, 352], "u8"), s, D([64, 576], "f16"), mode=2, G=32) == EDTYPE
    assert kd(L, c, s, D([64, 576], "f32")) == EDTYPE
    assert kd(L, c, s, D([64, 600], "bf16")) == ESHAPE    # d % 64
    assert kd(L, c, s, D([64, 64], "bf16")) == ESHAPE
    assert kd(L, c, D([63], "i32"), y) == ESHAPE
    assert kd(L, c, D([64], "f32"), y) == EDTYPE
    assert kd(L, c, s, y, mode=3) == EATTR
    assert kd(L, D([8, 16, 1, 1024], "u8"), s, y, mode=2, G=48) == EATTR
    assert kd(L, D([8, 16, 1, 671], "u8"), s, y) == ECAP  # headDim < kvCacheCol (672)
    assert kd(L, D([8, 16, 1, 672], "e4m3"), s, y) == EDTYPE
    assert kd(L, D([8, 16, 672], "u8"), s, y) == ENDIM
    assert kd(L, c, s, D([64, 576], "bf16", [1, 64])) == ELAYOUT
    assert kd(L, c, D([0], "i32"), D([0, 576], "bf16")) == OK


def test_indexer_validation(L):
    x, s = D([64, 128], "bf16"), D([64], "i32")
    c8, c4, sc = D([16, 8, 1, 128], "e4m3"), D([16, 8, 1, 64], "u8"), D([16, 8, 1, 4], "e8m0")
    f = lambda x, c, sc, s, m: L.kvq_indexer_quant_cache(R(x), R(c), R(sc), R(s), m, None)
    assert f(x, c8, sc, s, 0) == ENULL
    assert f(x, c4, sc, s, 3) == ENULL
    assert f(x, c8, D([16, 8, 1, 1], "f32"), s, 1) == ENULL
    assert f(x, c8, sc, s, 2) == EUNSUP                   # hifloat8
    assert f(x, c8, sc, s, 4) == EATTR
    assert f(x, c4, sc, s, 0) == EDTYPE                   # mxfp8 needs an fp8 cache
    assert f(x, c8, sc, s, 3) == EDTYPE                   # mxfp4 needs a uint8 cache
    assert f(x, c8, D([16, 8, 1, 4], "f32"), s, 0) == EDTYPE
    assert f(x, D([16, 8, 1, 127], "e4m3"), sc, s, 0) == ECAP
    assert f(x, D([16, 8, 1, 63], "u8"), sc, s, 3) == ECAP
    assert f(x, c8, D([16, 8, 1, 3], "e8m0"), s, 0) == ECAP
    assert f(x, c8, D([16, 4, 1, 4], "e8m0"), s, 0) == ESHAPE   # blockSize mismatch
    assert f(D([64, 128], "f32"), c8, sc, s, 0) == EDTYPE
    assert f(x, c8, sc, D([65], "i64"), 0) == ESHAPE


def rr(L, kv, g, c, s, idx, kc, cc, ks=None, cs=None, ko=None, co=None, mode=2):
    p = lambda t: None if t is None else R(t)
    return L.kvq_kv_rmsnorm_rope_cache(R(kv), R(g), R(c), R(s), R(idx), R(kc), R(cc), p(ks), p(cs), p(ko), p(co),
                                       ctypes.c_float(1e-6), mode, None)


def test_rmsnorm_rope_validation(L):
    kv, g = D([64, 1, 1, 576], "bf16"), D([512], "bf16")
    cs, sn, idx = D([64, 1, 1, 64], "bf16"), D([64, 1, 1, 64], "bf16"), D([64], "i32")
    kc, cc, sc = D([32, 128, 1, 64], "bf16"), D([32, 128, 1, 512], "e4m3"), D([1], "f32")
    assert rr(L, kv, g, cs, sn, idx, kc, cc, cs=sc) == ENULL
    assert rr(L, kv, g, cs, sn, idx, kc, cc) == ENULL               # quantised ckv without scale
    assert rr(L, kv, g, cs, sn, idx, kc, D([32, 128, 1, 512], "bf16")) == ENULL
    assert rr(L, D([64, 2, 1, 576], "bf16"), g, cs, sn, idx, kc, cc, cs=sc) == ESHAPE   # N must be 1
    assert rr(L, kv, g, cs, sn, idx, D([32, 128, 1, 63], "bf16"), cc, cs=sc) == ESHAPE  # Dk+Dv != D
    assert rr(L, kv, D([512], "f16"), cs, sn, idx, kc, cc, cs=sc) == EDTYPE
    assert rr(L, kv, g, cs, sn, idx, kc, cc, cs=sc, mode=4) == EUNSUP                  # PA_NZ
    assert rr(L, kv, g, cs, sn, idx, kc, cc, cs=sc, mode=7) == EATTR
    assert rr(L, kv, g, cs, sn, idx, D([32, 24, 1, 64], "bf16"), D([32, 24, 1, 512], "e4m3"),
              cs=sc) == ESHAPE                                                         # blockSize % 32
    assert rr(L, kv, g, cs, sn, idx, D([32, 128, 1, 64], "e5m2"), cc, ks=sc, cs=sc) == EDTYPE  # mixed fp8
    assert rr(L, kv, g, cs, sn, idx, kc, cc, cs=sc, co=sc) == EATTR                    # offset on fp8
    assert rr(L, kv, g, cs, sn, idx, kc, D([32, 128, 1, 512], "i8"), cs=sc, co=sc) == ENULL
    assert rr(L, kv, g, cs, sn, idx, kc, cc, cs=D([7], "f32")) == ESHAPE


def test_dequant_rope_quant_validation(L):
    x, c = D([16, 1024, 3072], "i32"), D([16, 1024, 1, 128], "bf16")
    kc = D([512, 128, 4, 128], "i8")
    ind, sk, ws = D([16384], "i32"), D([4, 128], "f32"), D([3072], "f32")
    q = D([16, 1024, 16, 128], "bf16")
    p = lambda t: None if t is None else R(t)

    def f(x=x, c=c, kc=kc, vc=kc, ind=ind, sk=sk, ws=ws, bias=None, splits=(2048, 512, 512), n=3, qm=0, lo=0,
          kvo=0, cm=1, q=q, ko=None, vo=None):
        arr = (ctypes.c_int64 * 3)(*splits)
        return L.kvq_dequant_rope_quant_kvcache(R(x), R(c), R(c), R(kc), R(vc), R(ind), R(sk), R(sk), None, None,
                                                p(ws), None, p(bias), arr, n, qm, lo, kvo, cm, R(q), p(ko), p(vo),
                                                None)
    assert f() == ENULL
    assert f(ws=None) == ENULL                              # int32 x needs weight_scale
    assert f(n=2) == EATTR
    assert f(splits=(2048, 512, 256)) == EATTR              # k and v splits differ
    assert f(splits=(2048, 256, 256)) == ESHAPE             # do not add up to H / Nkv
    assert f(qm=1) == EATTR and f(lo=1) == EATTR and f(cm=2) == EATTR
    assert f(x=D([16, 1024, 3072], "f32")) == EDTYPE
    assert f(x=D([16, 1024, 3072], "f16")) == EDTYPE         # 16-bit x must match cos
    assert f(x=D([16, 1024, 8, 3072], "i32")) == ENDIM
    assert f(x=D([16, 1024, 4160], "i32"), splits=(3136, 512, 512)) == ESHAPE   # tail > 4096
    assert f(kc=D([512, 128, 4, 128], "u8"), vc=D([512, 128, 4, 128], "u8")) == EDTYPE
    assert f(ind=D([16], "i32")) == ESHAPE                  # page mode: one index per token
    assert f(ind=D([16], "i32"), cm=0) == ESHAPE            # contiguous: cache too short for S=1024
    assert f(q=D([16, 1024, 15, 128], "bf16")) == ESHAPE
    assert f(kvo=1) == ENULL                                # kv_output needs k_out / v_out
    assert f(bias=D([3072], "i8")) == EDTYPE
    assert f(bias=D([3072], "bf16")) == ENULL
    kc48, s48 = D([512, 128, 4, 48], "i8"), D([4, 48], "f32")
    assert f(kc=kc48, vc=kc48, c=D([16, 1024, 1, 48], "bf16"), x=D([16, 1024, 1152], "i32"),
             splits=(768, 192, 192), q=D([16, 1024, 16, 48], "bf16"), sk=s48,
             ws=D([1152], "f32")) == ENULL   # D % 32 != 0 is supported
    kc24 = D([512, 128, 4, 24], "i8")
    assert f(kc=kc24, vc=kc24, c=D([16, 1024, 1, 24], "bf16"), x=D([16, 1024, 576], "i32"),
             splits=(288, 144, 144), q=D([16, 1024, 12, 24], "bf16")) == ESHAPE   # D % 16 != 0


def test_empty_inputs_are_accepted_whatever_their_strides(L):
    x, s, c = D([0, 576], "bf16", [0, 0]), D([0], "i32", [0]), D([8, 16, 1, 672], "u8")
    assert ce(L, x, s, c) == OK
    xi, si = D([0, 128], "f16", [0, 0]), D([0], "i64", [0])
    assert L.kvq_indexer_quant_cache(R(xi), R(D([16, 8, 1, 128], "e4m3")), R(D([16, 8, 1, 4], "e8m0")), R(si), 0,
                                     None) == OK


def test_missing_library_fails_loudly(tmp_path):
    """No CPU or library fallback: with libkvq.so absent the first call raises."""
    import subprocess
    import sys
    code = ("import kv_cache_quantize_b200 as kvq, torch\n"
            f"kvq.library_path = {str(tmp_path / 'absent.so')!r}\n"
            "x = torch.zeros((0, 128), dtype=torch.bfloat16)\n"
            "s = torch.zeros(0, dtype=torch.int32)\n"
            "c = torch.zeros((0, 16, 1, 224), dtype=torch.uint8)\n"
            "try:\n"
            "    kvq.kv_compress_epilog(x, s, c, 0)\n"
            "except RuntimeError as e:\n"
            "    print('raised:', e)\n"
            "else:\n"
            "    print('no error')\n")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT, timeout=300)
    assert "raised:" in out.stdout and "not built" in out.stdout, out.stdout + out.stderr


def test_row_widths_beyond_32_bit_indexing_are_rejected(L):
    """The indexer's d and the rmsnorm/rope D are bounded by 2^24 (the kernels index a row with 32-bit integers)."""
    wide = (1 << 24) + 32
    f = lambda x, c, sc, s: L.kvq_indexer_quant_cache(R(x), R(c), R(sc), R(s), 0, None)
    assert f(D([4, wide], "bf16"), D([1, 16, 1, wide], "e4m3"), D([1, 16, 1, wide // 32], "e8m0"),
             D([4], "i32")) == ESHAPE


def test_selftest_numbering(L):
    """Self-tests 0..10 exist; other numbers and a NULL result are rejected before any device work."""
    out = ctypes.c_uint64(0)
    assert L.kvq_selftest(11, ctypes.byref(out), None) == EATTR
    assert L.kvq_selftest(-1, ctypes.byref(out), None) == EATTR
    assert L.kvq_selftest(0, None, None) == ENULL


def test_host_tensors_are_rejected_before_any_launch():
    """A host tensor (or tensors on two devices) would make a kernel dereference a
    pointer it cannot use: the binding refuses the call instead."""
    x = torch.zeros((4, 128), dtype=torch.bfloat16)
    s = torch.zeros(4, dtype=torch.int32)
    c = torch.zeros((1, 16, 1, 224), dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA device"):
        kvq.kv_compress_epilog(x, s, c, 0)
    with pytest.raises(ValueError, match="CUDA device"):
        kvq.indexer_quant_cache(x, c, c, s, "mxfp8")
    with pytest.raises(ValueError, match="CUDA device"):
        kvq.kv_decompress(c, s, x, 0)


def test_calls_run_on_the_tensors_device(monkeypatch):
    """The library sizes grids and launches on the current device, so the binding
    makes the tensors' device current for the call when it is not already."""
    import contextlib
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    assert isinstance(kvq._on(torch.device("cuda", 0)), contextlib.nullcontext)
    assert isinstance(kvq._on(None), contextlib.nullcontext)
    ctx = kvq._on(torch.device("cuda", 1))
    assert isinstance(ctx, torch.cuda.device) and ctx.idx == 1


def test_check_flag_reports_fault_bits(monkeypatch, L):
    """check=True reads the fault word after the call and raises on a set bit."""
    calls = []

    def fake_get_error(stream, bits):
        calls.append(stream)
        ctypes.cast(bits, ctypes.POINTER(ctypes.c_uint32))[0] = kvq.FAULT_SLOT_RANGE
        return 0
    monkeypatch.setattr(L, "kvq_get_error", fake_get_error)
    with pytest.raises(kvq.KvqFault, match="FAULT_SLOT_RANGE"):
        kvq._faults("op", True, 1234)
    kvq._faults("op", False, 1234)
    assert calls == [1234]


def test_compressor_validation(L):
    x, wk, ape, out = D([2048, 1024], "bf16"), D([512, 1024], "bf16"), D([128, 512], "f32"), D([16, 512], "bf16")

    def f(x=x, wk=wk, wg=wk, ape=ape, out=out, ratio=128):
        return L.kvq_compressor(R(x), R(wk), R(wg), R(ape), R(out), ratio, None)
    assert f() == ENULL                                              # valid; stops at the NULL data
    assert f(ratio=96) == EATTR and f(ratio=1) == EATTR and f(ratio=256) == EATTR
    assert f(x=D([2048, 1024], "f16")) == EDTYPE and f(ape=D([128, 512], "bf16")) == EDTYPE
    assert f(x=D([2048, 1000], "bf16"), wk=D([512, 1000], "bf16")) == ESHAPE      # H % 512
    assert f(x=D([2048, 512], "bf16"), wk=D([512, 512], "bf16")) == ESHAPE        # H < 1024
    assert f(wk=D([256, 1024], "bf16"), wg=D([256, 1024], "bf16"), ape=D([128, 256], "f32"),
             out=D([16, 256], "bf16")) == ESHAPE                                   # D is 128 or 512
    assert f(x=D([2000, 1024], "bf16"), out=D([15, 512], "bf16")) == ESHAPE       # T % cmp_ratio
    assert f(out=D([15, 512], "bf16")) == ESHAPE and f(ape=D([64, 512], "f32")) == ESHAPE
    assert f(wk=D([512, 1024], "bf16", [2048, 1])) == ELAYOUT
    assert f(x=D([2, 1024, 1024], "bf16"), out=D([16, 512], "bf16")) == ENULL     # leading dims are tokens
    assert f(x=D([0, 1024], "bf16"), out=D([0, 512], "bf16")) == OK               # nothing to do
    assert f(x=D([2048, 1024], "bf16"), wk=D([128, 1024], "bf16"), wg=D([128, 1024], "bf16"),
             ape=D([128, 128], "f32"), out=D([16, 128], "bf16")) == ENULL          # D = 128
    # C4A / C4Li: weights of 2 D rows, Ape [4, 2 D], cmp_ratio 4
    w2, a2, o4 = D([1024, 1024], "bf16"), D([4, 1024], "f32"), D([512, 512], "bf16")
    assert f(wk=w2, wg=w2, ape=a2, out=o4, ratio=4) == ENULL                       # C4A, valid
    assert f(wk=D([256, 1024], "bf16"), wg=D([256, 1024], "bf16"), ape=D([4, 256], "f32"),
             out=D([512, 128], "bf16"), ratio=4) == ENULL                           # C4Li, valid
    assert f(wk=w2, wg=w2, ape=D([128, 1024], "f32"), out=out, ratio=128) == EATTR  # coff 2 needs ratio 4
    assert f(wk=w2, wg=wk, ape=a2, out=o4, ratio=4) == ESHAPE                      # gate rows differ
    assert f(wk=w2, wg=w2, ape=D([4, 512], "f32"), out=o4, ratio=4) == ESHAPE      # Ape [4, 2 D]
    assert f(wk=D([768, 1024], "bf16"), wg=D([768, 1024], "bf16"), ape=D([4, 768], "f32"), out=o4,
             ratio=4) == ESHAPE                                                    # rows neither D nor 2 D
