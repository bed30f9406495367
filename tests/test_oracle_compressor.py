"""Pins of the Compressor oracle (oracle/compressor.py), CPU only.

Source: aclnnCompressor, 计算公式 steps 1-5, C128A form (coff = 1).  Each pin
checks the oracle against something other than itself: hand-worked examples,
closed forms (group mean, softmax weights of a per-row Ape with no gate),
limits (a dominant Ape entry selects one row) and invariants that the
formula fixes (a per-channel shift of the scores changes nothing; a
permutation of a group's rows with Ape's rows changes nothing; groups are
independent; every output channel is a convex combination of its group's
kv_state values).  Each pin is a function of the oracle module, so that
tests/test_oracle_mutations.py can run the same pins against copies with a
planted mistake.
"""
import math

import numpy as np
import pytest

import oracle.compressor as ORACLE
from _golden import read_cases


def bf16_bits(a) -> np.ndarray:
    """float values -> bf16 bit patterns by round to nearest even (inputs in the
    pins are chosen exact in bf16 or are random values whose rounding only has
    to be deterministic)."""
    u = np.ascontiguousarray(np.asarray(a, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def exact(bits) -> np.ndarray:
    """Exact values of bf16 bit patterns, written independently of the oracle."""
    return np.array([float(np.array([int(b) << 16], dtype=np.uint32).view(np.float32)[0])
                     for b in np.asarray(bits).ravel()]).reshape(np.asarray(bits).shape)


def _mat(text):
    return np.array([[float(v) for v in row.split()] for row in text.split(";")])


def _rand(seed, T, H, D, ratio, ape_scale=1.0):
    rng = np.random.default_rng(seed)
    x = bf16_bits(rng.standard_normal((T, H)))
    wk = bf16_bits(rng.standard_normal((D, H)) / math.sqrt(H))
    wg = bf16_bits(rng.standard_normal((D, H)) / math.sqrt(H))
    ape = (rng.standard_normal((ratio, D)) * ape_scale).astype(np.float32)
    return x, wk, wg, ape


def _kv(x, wk):
    """kv_state by explicit sums over H, independent of the oracle's matmul."""
    X, W = exact(x), exact(wk)
    return np.einsum("th,dh->td", X, W)


# ---------------------------------------------------------------------------
def pin_worked_examples(C):
    for name, case in read_cases("compressor_examples.txt").items():
        ratio = int(case["ratio"])
        x = bf16_bits(_mat(case["x"]))
        wk, wg = bf16_bits(_mat(case["w_kv"])), bf16_bits(_mat(case["w_gate"]))
        ape = _mat(case["ape"]).astype(np.float32)
        want = _mat(case["out"])
        got = C.compressor(x, wk, wg, ape, ratio)
        assert got.shape == want.shape, name
        assert np.allclose(got, want, rtol=1e-13, atol=1e-13), (name, got, want)


def pin_group_mean(C):
    """W^Gate = 0, Ape = 0: equal weights, C = mean of the group's kv_state rows,
    computed here as (mean of the group's x rows) @ W^KV^T."""
    for ratio, D in ((4, 3), (8, 5), (128, 2)):
        x, wk, _, _ = _rand(ratio, 3 * ratio, 16, D, ratio)
        got = C.compressor(x, wk, np.zeros_like(wk), np.zeros((ratio, D), np.float32), ratio)
        want = exact(x).reshape(3, ratio, 16).mean(axis=1) @ exact(wk).T
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def pin_row_selection(C):
    """A dominant Ape entry at (row r_c, channel c) gives C[g, c] = kv_state of
    row r_c of group g (the other weights are below e^-150 relative)."""
    ratio, D, G = 8, 6, 3
    x, wk, wg, _ = _rand(7, G * ratio, 12, D, ratio)
    pick = np.array([5, 0, 7, 2, 2, 6])
    ape = np.zeros((ratio, D), np.float32)
    ape[pick, np.arange(D)] = 300.0
    got = C.compressor(x, wk, wg, ape, ratio)
    kv = _kv(x, wk)
    for g in range(G):
        for c in range(D):
            assert got[g, c] == pytest.approx(kv[g * ratio + pick[c], c], rel=1e-12, abs=1e-12)


def pin_row_weights_closed_form(C):
    """W^Gate = 0 and Ape[r, c] = u_r for every channel: the weights are
    exp(u_r) / sum_s exp(u_s), the same for every channel and group."""
    ratio, D, G = 16, 4, 2
    x, wk, _, _ = _rand(11, G * ratio, 8, D, ratio)
    u = np.linspace(-2.0, 3.0, ratio).astype(np.float32)
    ape = np.repeat(u[:, None], D, axis=1)
    got = C.compressor(x, wk, np.zeros_like(wk), ape, ratio)
    w = [math.exp(float(v)) for v in u]
    z = sum(w)
    kv = _kv(x, wk)
    for g in range(G):
        for c in range(D):
            want = sum(w[r] / z * kv[g * ratio + r, c] for r in range(ratio))
            assert got[g, c] == pytest.approx(want, rel=1e-12, abs=1e-12)


def pin_channel_shift_invariance(C):
    """Adding one constant per channel to Ape leaves every output unchanged
    (the softmax runs over rows, channel by channel)."""
    ratio, D = 8, 5
    x, wk, wg, ape = _rand(13, 4 * ratio, 16, D, ratio, ape_scale=2.0)
    base = C.compressor(x, wk, wg, ape, ratio)
    # the shift is applied in float64, where it is exact (in float32 it would round)
    shifted = C.compressor(x, wk, wg, ape.astype(np.float64) + np.array([3.0, -7.0, 0.5, 11.0, -2.0])[None, :],
                           ratio)
    assert np.allclose(base, shifted, rtol=1e-11, atol=1e-11)


def pin_permutation_equivariance(C):
    """Permuting the rows inside every group together with Ape's rows leaves C unchanged."""
    ratio, D, G = 8, 4, 3
    x, wk, wg, ape = _rand(17, G * ratio, 16, D, ratio, ape_scale=1.5)
    perm = np.array([3, 7, 0, 5, 1, 6, 2, 4])
    rows = np.concatenate([g * ratio + perm for g in range(G)])
    a = C.compressor(x, wk, wg, ape, ratio)
    b = C.compressor(x[rows], wk, wg, ape[perm], ratio)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


def pin_group_locality(C):
    """Each output row depends on its own group's rows only, and on all of them."""
    ratio, D, G = 4, 3, 3
    x, wk, wg, ape = _rand(19, G * ratio, 8, D, ratio)
    a = C.compressor(x, wk, wg, ape, ratio)
    x2 = x.copy()
    x2[ratio:2 * ratio] = bf16_bits(np.random.default_rng(23).standard_normal((ratio, 8)))
    b = C.compressor(x2, wk, wg, ape, ratio)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[2], b[2])
    assert not np.allclose(a[1], b[1])
    for r in range(ratio):       # every row of the group moves its output
        x3 = x.copy()
        x3[ratio + r] = bf16_bits(np.full(8, 2.0))
        assert not np.allclose(C.compressor(x3, wk, wg, ape, ratio)[1], a[1])


def pin_convexity(C):
    ratio, D, G = 32, 8, 2
    x, wk, wg, ape = _rand(29, G * ratio, 16, D, ratio, ape_scale=3.0)
    got = C.compressor(x, wk, wg, ape, ratio)
    kv = _kv(x, wk).reshape(G, ratio, D)
    assert np.all(got >= kv.min(axis=1) - 1e-12) and np.all(got <= kv.max(axis=1) + 1e-12)


def pin_selected_groups(C):
    """The group-subset form returns exactly the listed rows of the full result."""
    ratio, D, G = 8, 4, 5
    x, wk, wg, ape = _rand(31, G * ratio, 16, D, ratio)
    full = C.compressor(x, wk, wg, ape, ratio)
    sub = C.compressor(x, wk, wg, ape, ratio, groups=[4, 1])
    assert np.array_equal(sub, full[[4, 1]])


PINS = [pin_worked_examples, pin_group_mean, pin_row_selection, pin_row_weights_closed_form,
        pin_channel_shift_invariance, pin_permutation_equivariance, pin_group_locality, pin_convexity,
        pin_selected_groups]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_compressor_oracle_pin(pin):
    pin(ORACLE)


def test_bf16_helper_is_exact():
    """The tests' own bf16 rounding: exact values survive, ties go to even."""
    vals = np.array([1.0, -2.5, 3.0, 0.0078125, 1 + 2 ** -7], dtype=np.float32)
    assert np.array_equal(exact(bf16_bits(vals)), vals.astype(np.float64))
    assert exact(bf16_bits(np.float32([1 + 2 ** -8])))[0] == 1.0              # tie -> even
    assert exact(bf16_bits(np.float32([1 + 3 * 2 ** -8])))[0] == 1 + 2 ** -6  # tie -> even (up)
