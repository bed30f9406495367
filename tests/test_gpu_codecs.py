"""Device codecs against the oracle's, over every finite bf16 value x scales and
millions of random binary32 values (checks the cvt operand order, the sign of
zero, saturation and subnormals of the hardware conversions)."""
import numpy as np
import pytest
import torch

import kv_cache_quantize_b200 as kvq
import oracle

pytestmark = pytest.mark.gpu


def _inputs(seed: int, nonneg: bool = False) -> np.ndarray:
    bits = np.arange(1 << 16, dtype=np.uint32)
    bits = bits[(bits & 0x7F80) != 0x7F80]
    bf = (bits << 16).astype(np.uint32).view(np.float32)
    scales = np.array([2.0 ** k for k in (-140, -133, -126, -20, -9, -6, -1, 0, 1, 3, 7, 14, 30, 100)]
                      + [1 / 448, 1 / 6, 1 / 57344, 0.1, 3.7, 64.0, 1e-40], dtype=np.float32)
    with np.errstate(over="ignore"):
        v = (bf[:, None] * scales[None, :]).astype(np.float32).ravel()
    rng = np.random.default_rng(seed)
    rnd = rng.integers(0, 1 << 32, size=4_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    with np.errstate(invalid="ignore"):
        near = (rnd % np.float32(1000.0)).astype(np.float32)
    v = np.concatenate([v, rnd, near, np.array([0.0, -0.0, 1e-45, -1e-45, 448.0, 464.0, 480.0, -500.0,
                                                6.0, 5.0, 7.0, 0.25, 0.75, 57344.0, 61440.0], np.float32)])
    v = v[np.isfinite(v)]
    if nonneg:
        v = np.abs(v)
    return v


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2", "e2m1"])
def test_fp_codes_match_oracle(fmt):
    v = _inputs(1)
    got = kvq.convert(fmt, torch.from_numpy(v).cuda()).cpu().numpy().astype(np.uint32)
    want = oracle.encode(fmt, v)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches; first v={v[bad[0]]!r} gpu={got[bad[0]]:#x} oracle={want[bad[0]]:#x}"


def test_bf16_rounding_matches_oracle():
    v = _inputs(2)
    got = kvq.convert("bf16", torch.from_numpy(v).cuda()).cpu().numpy().view(np.uint16).astype(np.uint32)
    assert np.array_equal(got, oracle.encode("bf16", v, saturate=False))


def test_e8m0_ceil_matches_oracle():
    v = _inputs(3, nonneg=True)
    got = kvq.convert("e8m0", torch.from_numpy(v).cuda()).cpu().numpy()
    assert np.array_equal(got, oracle.e8m0_ceil(v))


def test_int8_static_matches_oracle():
    v = np.concatenate([_inputs(4), np.arange(-200.5, 200.5, 0.5, dtype=np.float32)])
    got = kvq.convert("i8", torch.from_numpy(v).cuda()).cpu().numpy().view(np.int8)
    assert np.array_equal(got, oracle.int8_static(v))
