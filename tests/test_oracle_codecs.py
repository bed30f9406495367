"""Pins of the oracle's number-format codecs (CPU only).

Each codec of oracle/kvq_oracle.c is checked against something other than
itself: the published code tables (tests/golden/format_codes.txt), a
nearest-value search over the enumerated format (tests/_formats.py),
library conversions (torch, numpy, ml_dtypes) and exact rational arithmetic.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from _formats import decode as t_decode
from _formats import max_finite, nearest_code
from _golden import read_table

FP_FMTS = ["e4m3", "e5m2", "e2m1"]


def all_finite_bf16() -> np.ndarray:
    bits = np.arange(1 << 16, dtype=np.uint32)
    bits = bits[(bits & 0x7F80) != 0x7F80]
    return (bits << 16).astype(np.uint32).view(np.float32)


def random_finite_f32(n: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 1 << 32, size=n, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    return v[np.isfinite(v)]


SCALES = np.array([2.0 ** k for k in (-140, -133, -126, -20, -9, -6, -1, 0, 1, 3, 7, 14, 30, 100)]
                  + [1 / 448, 1 / 6, 1 / 57344, 0.1, 3.7, 64.0, 1e-40], dtype=np.float32)


@pytest.mark.parametrize("fmt", FP_FMTS)
def test_encode_equals_nearest_search_all_bf16_times_scales(fmt):
    with np.errstate(over="ignore"):
        v = (all_finite_bf16()[:, None] * SCALES[None, :]).astype(np.float32).ravel()
    v = v[np.isfinite(v)]
    got = oracle.encode(fmt, v)
    want = nearest_code(fmt, v)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{fmt}: {bad.size} mismatches, first v={v[bad[0]]!r} got={got[bad[0]]:#x} want={want[bad[0]]:#x}"


@pytest.mark.parametrize("fmt", FP_FMTS)
def test_encode_equals_nearest_search_random_f32(fmt):
    v = random_finite_f32(2_000_000, seed=11)
    # bring a share of the values into the format's range so every binade is exercised
    near = (random_finite_f32(2_000_000, seed=12) % np.float32(2 * max_finite(fmt))).astype(np.float32)
    v = np.concatenate([v, near])
    assert np.array_equal(oracle.encode(fmt, v), nearest_code(fmt, v))


@pytest.mark.parametrize("fmt,tdt", [("e4m3", torch.float8_e4m3fn), ("e5m2", torch.float8_e5m2)])
def test_encode_matches_torch_cast_in_range(fmt, tdt):
    v = np.concatenate([random_finite_f32(1_000_000, 21), all_finite_bf16()])
    v = v[np.abs(v) <= max_finite(fmt)]
    ref = torch.from_numpy(v).to(tdt).view(torch.uint8).numpy().astype(np.uint32)
    assert np.array_equal(oracle.encode(fmt, v), ref)


def test_e2m1_matches_ml_dtypes():
    ml_dtypes = pytest.importorskip("ml_dtypes")
    if not hasattr(ml_dtypes, "float4_e2m1fn"):
        pytest.skip("ml_dtypes without float4_e2m1fn")
    v = np.concatenate([random_finite_f32(500_000, 31) % np.float32(6.0), all_finite_bf16()])
    v = v[np.abs(v) <= 6.0].astype(np.float32)
    ref = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8).astype(np.uint32) & 0xF
    assert np.array_equal(oracle.encode("e2m1", v), ref)


def test_golden_code_values():
    for row in read_table("format_codes.txt"):
        fmt, a, b = row[0], row[1], row[2]
        if fmt == "e2m1_rne":
            assert oracle.encode("e2m1", [float(a)])[0] == int(b, 16), row
            continue
        code, value = int(a, 16), float(b)
        dec = oracle.decode(fmt, [code])[0]
        assert dec == np.float32(value) and np.signbit(dec) == np.signbit(value), row
        if fmt == "bf16":
            assert oracle.encode("bf16", [value], saturate=False)[0] == code, row
        else:
            assert oracle.encode(fmt, [value])[0] == code, row


@pytest.mark.parametrize("fmt", FP_FMTS)
def test_decode_matches_definition_and_roundtrips(fmt):
    nbits = {"e4m3": 8, "e5m2": 8, "e2m1": 4}[fmt]
    codes = np.arange(1 << nbits, dtype=np.uint32)
    dec = oracle.decode(fmt, codes)
    ref = t_decode(fmt, codes).astype(np.float32)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isnan(dec), np.isnan(ref))
    assert np.array_equal(dec[fin], ref[fin])
    # every finite code is reproduced by encoding its own value (sign of zero included)
    assert np.array_equal(oracle.encode(fmt, dec[fin]), codes[fin])


@pytest.mark.parametrize("fmt", FP_FMTS)
def test_encode_is_monotone_and_saturates(fmt):
    v = np.sort(np.concatenate([random_finite_f32(200_000, 41), all_finite_bf16()]))
    dec = oracle.decode(fmt, oracle.encode(fmt, v))
    assert np.all(np.diff(dec.astype(np.float64)) >= 0)
    m = max_finite(fmt)
    assert np.all(np.abs(dec) <= m)
    big = np.array([m * 1.01, 1e30, 3.4e38, -3.4e38], dtype=np.float32)
    assert np.array_equal(np.abs(oracle.decode(fmt, oracle.encode(fmt, big))), np.full(4, m, np.float32))


def test_bf16_rounding_matches_torch():
    v = np.concatenate([random_finite_f32(2_000_000, 51),
                        np.array([0.0, -0.0, 1e-45, -1e-45, 3.3895e38, 1.0000001], np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.encode("bf16", v, saturate=False), ref.astype(np.uint32))


def test_f16_rounding_matches_numpy():
    v = np.concatenate([random_finite_f32(2_000_000, 52) % np.float32(70000.0),
                        np.array([0.0, -0.0, 6e-8, 65504.0, 65520.0, 1e5], np.float32)])
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16).astype(np.uint32)
        assert np.array_equal(oracle.encode("f16", v, saturate=False), ref)
        assert np.array_equal(oracle.decode("f16", ref), v.astype(np.float16).astype(np.float32))


@pytest.mark.parametrize("fp_max", [448.0, 57344.0, 6.0])
def test_e8m0_ceil_is_the_exact_power_of_two_bound(fp_max):
    a = all_finite_bf16()
    a = a[a > 0]
    q = (a / np.float32(fp_max)).astype(np.float32)        # IEEE binary32 division (numpy)
    b = oracle.e8m0_ceil(q)
    fm = Fraction(fp_max)
    for ai, bi in zip(a.tolist(), b.tolist()):
        ratio = Fraction(ai) / fm                          # the exact quotient, not the rounded one
        assert Fraction(2) ** (bi - 127) >= ratio
        assert bi == 0 or Fraction(2) ** (bi - 128) < ratio
    assert oracle.e8m0_ceil([0.0])[0] == 0


def test_e8m0_scaled_values_never_exceed_fp_max():
    # consequence of the bound: |a * 2^(127-b)| <= FP_MAX for every bf16 amax
    a = all_finite_bf16()
    a = a[a > 0]
    for fp_max in (448.0, 57344.0, 6.0):
        b = oracle.e8m0_ceil((a / np.float32(fp_max)).astype(np.float32)).astype(np.int64)
        scaled = a.astype(np.float64) * np.exp2(127.0 - b)
        assert np.all(scaled <= fp_max)


def test_int8_static_matches_numpy_rint_clip():
    rng = np.random.default_rng(61)
    v = np.concatenate([rng.uniform(-300, 300, 1_000_000).astype(np.float32),
                        np.arange(-140.5, 140.5, 0.5, dtype=np.float32),
                        np.array([1e30, -1e30, np.inf, -np.inf], np.float32)])
    ref = np.clip(np.rint(v), -128, 127).astype(np.int8)
    assert np.array_equal(oracle.int8_static(v), ref)
    assert oracle.int8_static([np.nan])[0] == 0
