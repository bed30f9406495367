"""Pins of the oracle's packed-row decoder (CPU only).

The decoder is the inverse of kv_compress_epilog: code value x group scale,
rounded once to bf16 (the rope of modes 0/1 is stored bf16; in mode 2 it is
the FP8 code divided by xScale).  What pins it:
  * exactness     -- rows built from values that the encoding represents
                     exactly (each group's maximum is FP_MAX * 2^k, so the
                     stored scale is 2^k and every x / scale is a code value)
                     must come back bit for bit;
  * error bound   -- on random rows (outliers included) every decoded value
                     lies within half a code step (in the group's scale) plus
                     half a bf16 ulp of x, which fails for a wrong scale
                     index, nibble order, segment offset or sign;
  * skip / fault  -- rows of skipped tokens keep y's contents; an out-of-range
                     slot raises the fault bit and leaves its row alone.
The expected values come from the test-side format tables (_formats), not
from the oracle's own codecs.
"""
import numpy as np
import pytest

import oracle
from _formats import code_value, positive_table
from _oracle_harness import paged
from kv_cache_quantize_b200 import workloads as W

FP_MAX = {"e4m3": 448.0, "e2m1": 6.0}


def _bits_to_f64(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def _cache_for(T, d, mode, G, extra=8, seed=0):
    col = oracle.kv_cache_col(d, mode, G)
    nblk = max(1, (2 * T + 15) // 16)
    return W.make_cache(np.random.default_rng(seed), nblk, 16, col + extra, 1, 1, 24)


def _roundtrip(x_bits, mode, G, x_scale, slots, cache, y0=None):
    T, d = x_bits.shape
    st = cache.storage.copy()
    f = oracle.kv_compress_epilog(x_bits, slots, paged(cache, st), mode, G, x_scale)
    assert f == 0
    y, f2 = oracle.kv_decompress(paged(cache, st), slots, d, mode, G, x_scale, y=y0)
    return y, f2


def _representable_rows(rng, T, d, mode, G, m_rope):
    """bf16 rows whose every group is exactly representable by the encoding."""
    n = d - 64
    fmt = "e2m1" if mode == 2 else "e4m3"
    _, vals = positive_table(fmt)
    vals = vals[vals <= FP_MAX[fmt]]
    g = G if mode == 2 else 64
    x = np.zeros((T, d), dtype=np.float64)
    for t in range(T):
        for j in range(n // g):
            k = int(rng.integers(-24, 12))
            v = rng.choice(vals, size=g) * rng.choice([-1.0, 1.0], size=g)
            v[int(rng.integers(0, g))] = FP_MAX[fmt] * rng.choice([-1.0, 1.0])
            x[t, j * g:(j + 1) * g] = v * 2.0 ** k
        if mode == 2:
            _, rv = positive_table("e4m3")
            x[t, n:] = rng.choice(rv[rv <= 448.0], size=64) * rng.choice([-1.0, 1.0], size=64) * 2.0 ** -m_rope
        else:
            x[t, n:] = rng.standard_normal(64)
    bits = W.to_bf16_bits(x.astype(np.float32))
    assert np.array_equal(_bits_to_f64(bits)[:, :n], x[:, :n])     # the construction is exact in bf16
    return bits


@pytest.mark.parametrize("mode,G", [(0, 64), (1, 64), (2, 16), (2, 32), (2, 64)])
@pytest.mark.parametrize("d", [128, 576])
def test_roundtrip_is_exact_on_representable_rows(mode, G, d):
    rng = np.random.default_rng(100 + 7 * mode + G + d)
    T = 24
    m_rope = 3
    x = _representable_rows(rng, T, d, mode, G, m_rope)
    slots = rng.choice(2 * T, T, replace=False).astype(np.int32)
    y, f = _roundtrip(x, mode, G, 2.0 ** m_rope, slots, _cache_for(T, d, mode, G))
    assert f == 0
    assert np.array_equal(y, x)


def _half_step(fmt, v):
    """Half the spacing of the format's grid around |v| (v in code units)."""
    _, vals = positive_table(fmt)
    a = np.abs(v)
    i = np.clip(np.searchsorted(vals, a), 1, len(vals) - 1)
    return (vals[i] - vals[i - 1]) / 2.0


@pytest.mark.parametrize("mode,G", [(0, 64), (1, 64), (2, 16), (2, 32), (2, 64)])
def test_roundtrip_error_bound_on_random_rows(mode, G):
    T, d, xs = 200, 576, 0.1
    case = W.gen_compress("rt", T=T, d=d, quant_mode=mode, num_blocks=32, block_size=16,
                          head_dim=oracle.kv_cache_col(d, mode, G) + 5, group_size=G, x_scale=xs,
                          skip_frac=0.1, outlier_frac=0.05, seed=3)
    x_bits, slots = case.arrays["x"], case.arrays["slot_mapping"]
    y, f = _roundtrip(x_bits, mode, G, np.float32(xs), slots, case.caches["cache"])
    assert f == 0
    n = d - 64
    x = _bits_to_f64(x_bits)
    yv = _bits_to_f64(y)
    live = slots != -1
    assert live.sum() > 0
    g = G if mode == 2 else 64
    fmt = "e2m1" if mode == 2 else "e4m3"
    xg = np.abs(x[:, :n]).reshape(T, n // g, g)
    amax = xg.max(axis=2)
    if mode == 1:
        scale = 2.0 ** np.ceil(np.log2(np.maximum(amax / 448.0, 2.0 ** -127)))
    else:
        scale = _bits_to_f64(W.to_bf16_bits((amax / FP_MAX[fmt]).astype(np.float32)))
    s = np.repeat(scale, g, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s > 0, x[:, :n] / s, 0.0)
    bound = s * _half_step(fmt, v) * (1 + 2.0 ** -20) + np.abs(yv[:, :n]) * 2.0 ** -8
    err = np.abs(yv[:, :n] - x[:, :n])
    assert np.all(err[live] <= bound[live] + 1e-300)
    if mode == 2:
        r = x[:, n:] * float(np.float32(xs))
        rb = _half_step("e4m3", r) / float(np.float32(xs)) * (1 + 2.0 ** -20) + np.abs(yv[:, n:]) * 2.0 ** -8
        assert np.all(np.abs(yv[:, n:] - x[:, n:])[live] <= rb[live])
    else:
        assert np.array_equal(y[live, n:], x_bits[live, n:])
    # the bound is tight enough to matter: a decoder that dropped the scale would fail it
    assert np.any(np.abs(yv[:, :n] / np.where(s > 0, s, 1) - x[:, :n])[live] > bound[live])


def test_skipped_rows_untouched_and_bad_slot_faults():
    T, d = 10, 128
    case = W.gen_compress("sk", T=T, d=d, quant_mode=0, num_blocks=2, block_size=16,
                          head_dim=oracle.kv_cache_col(d, 0, 64), seed=5)
    slots = case.arrays["slot_mapping"].copy()
    st = case.caches["cache"].storage.copy()
    oracle.kv_compress_epilog(case.arrays["x"], slots, paged(case.caches["cache"], st), 0)
    slots[2] = -1
    slots[5] = 32          # past the 2 x 16 slots
    y0 = np.full((T, d), 0x7E57, dtype=np.uint16)
    y, f = oracle.kv_decompress(paged(case.caches["cache"], st), slots, d, 0, 64, 1.0, y=y0.copy())
    assert f == 1
    assert np.all(y[2] == 0x7E57) and np.all(y[5] == 0x7E57)
    others = [t for t in range(T) if t not in (2, 5)]
    assert not np.any(y[others] == 0x7E57)


def test_decoded_codes_follow_the_format_tables():
    """A row of single-code groups decodes to code value x scale for every E4M3 code."""
    d = 128
    codes = np.arange(256, dtype=np.uint8)
    codes = codes[np.isfinite([code_value("e4m3", int(c)) for c in codes])]
    for c0 in range(0, len(codes), 64):
        chunk = codes[c0:c0 + 64]
        row = np.zeros(oracle.kv_cache_col(d, 0, 64), dtype=np.uint8)
        row[:len(chunk)] = chunk
        row[64 + 128:64 + 130] = np.frombuffer(np.uint16(0x4040).tobytes(), dtype=np.uint8)   # scale 3.0
        cache = W.make_cache(np.random.default_rng(0), 1, 1, row.size, 1, 1, 0)
        cache.storage[cache.offset:cache.offset + row.size] = row
        y, _ = oracle.kv_decompress(paged(cache, cache.storage), np.array([0]), d, 0)
        want = np.array([code_value("e4m3", int(c)) * 3.0 for c in chunk])
        got = _bits_to_f64(y[0, :len(chunk)])
        assert np.array_equal(got, _bits_to_f64(W.to_bf16_bits(want.astype(np.float32)))), c0


@pytest.mark.parametrize("mode", [0, 1])
def test_f16_roundtrip_keeps_the_rope_and_bounds_the_codes(mode):
    """float16 x (quantMode 0/1): decoding into float16 gives back the rope bit for bit
    (it is stored unchanged) and every nope value within half a code step in its group's
    scale plus half an f16 ulp; exactly representable rows come back exactly."""
    T, d = 120, 320
    rng = np.random.default_rng(40 + mode)
    xf = (rng.standard_normal((T, d)) * 20).astype(np.float16)
    x_bits = xf.view(np.uint16)
    slots = rng.choice(2 * T, T, replace=False).astype(np.int32)
    slots[::9] = -1
    cache = _cache_for(T, d, mode, 64, seed=5)
    st = cache.storage.copy()
    assert oracle.kv_compress_epilog(x_bits, slots, paged(cache, st), mode, 64, 1.0, x_dtype="f16") == 0
    y, f = oracle.kv_decompress(paged(cache, st), slots, d, mode, 64, 1.0, y_dtype="f16")
    assert f == 0
    live = slots != -1
    n = d - 64
    assert np.array_equal(y[live, n:], x_bits[live, n:])
    x = xf.astype(np.float64)
    yv = y.view(np.float16).astype(np.float64)
    amax = np.abs(x[:, :n]).reshape(T, n // 64, 64).max(axis=2)
    if mode == 1:
        scale = 2.0 ** np.ceil(np.log2(np.maximum(amax / 448.0, 2.0 ** -127)))
    else:
        scale = _bits_to_f64(W.to_bf16_bits((amax / 448.0).astype(np.float32)))
    s = np.repeat(scale, 64, axis=1)
    v = np.where(s > 0, x[:, :n] / s, 0.0)
    bound = s * _half_step("e4m3", v) * (1 + 2.0 ** -20) + np.abs(yv[:, :n]) * 2.0 ** -11
    assert np.all(np.abs(yv[:, :n] - x[:, :n])[live] <= bound[live])
    # and the decoder refuses float16 output in quantMode 2 (bfloat16 x only there)
    with pytest.raises(Exception):
        oracle.kv_decompress(paged(cache, st), slots, d, 2, 32, 0.1, y_dtype="f16")
