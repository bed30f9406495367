"""Pins of the Compressor oracle (oracle/compressor.py), CPU only.

Source: aclnnCompressor, 计算公式 steps 1-5, C128A form (coff = 1) and C4A
form (coff = 2, cmp_ratio = 4).  Each pin
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


# ---------------------------------------------------------------------------
# C4A form (coff = 2, cmp_ratio = 4): group i = the a projections of its own
# four tokens and the b projections of the next group's four
# ---------------------------------------------------------------------------
def _rand_c4a(seed, G, H, D, ape_scale=1.0):
    rng = np.random.default_rng(seed)
    x = bf16_bits(rng.standard_normal((4 * G, H)))
    wk = bf16_bits(rng.standard_normal((2 * D, H)) / math.sqrt(H))
    wg = bf16_bits(rng.standard_normal((2 * D, H)) / math.sqrt(H))
    ape = (rng.standard_normal((4, 2 * D)) * ape_scale).astype(np.float32)
    return x, wk, wg, ape


def pin_c4a_eight_row_mean(C):
    """W^Gate = 0, Ape = 0: equal weights over a group's eight rows, so C_i =
    (mean of its own four x rows @ W^aKV^T + mean of the next four @ W^bKV^T) / 2;
    the last group has only its own four rows: C = mean of them @ W^aKV^T."""
    G, H, D = 5, 16, 3
    x, wk, _, _ = _rand_c4a(37, G, H, D)
    got = C.compressor_c4a(x, wk, np.zeros_like(wk), np.zeros((4, 2 * D), np.float32))
    X = exact(x).reshape(G, 4, H).mean(axis=1)
    Wa, Wb = exact(wk)[:D], exact(wk)[D:]
    for i in range(G - 1):
        assert np.allclose(got[i], (X[i] @ Wa.T + X[i + 1] @ Wb.T) / 2, rtol=1e-12, atol=1e-12)
    assert np.allclose(got[G - 1], X[G - 1] @ Wa.T, rtol=1e-12, atol=1e-12)


def pin_c4a_selects_an_a_row(C):
    """A dominant entry of Ape's a columns, Ape[p_c, c], selects kv^a of token
    4i + p_c for channel c in every group (the last one included)."""
    G, H, D = 4, 12, 5
    x, wk, wg, _ = _rand_c4a(41, G, H, D)
    pick = np.array([3, 0, 2, 1, 3])
    ape = np.zeros((4, 2 * D), np.float32)
    ape[pick, np.arange(D)] = 300.0
    got = C.compressor_c4a(x, wk, wg, ape)
    kv_a = _kv(x, wk[:D])
    for i in range(G):
        for c in range(D):
            assert got[i, c] == pytest.approx(kv_a[4 * i + pick[c], c], rel=1e-12, abs=1e-12)


def pin_c4a_selects_a_b_row(C):
    """A dominant entry of Ape's b columns, Ape[p_c, D + c], selects kv^b of
    token 4(i + 1) + p_c (the next group's) for channel c; the last group,
    with no next four tokens, is the four-row softmax of its own a rows
    (the C128A form with cmp_ratio 4, pinned above, on those rows)."""
    G, H, D = 4, 12, 5
    x, wk, wg, _ = _rand_c4a(43, G, H, D)
    pick = np.array([1, 3, 0, 2, 2])
    ape = np.zeros((4, 2 * D), np.float32)
    ape[pick, D + np.arange(D)] = 300.0
    got = C.compressor_c4a(x, wk, wg, ape)
    kv_b = _kv(x, wk[D:])
    for i in range(G - 1):
        for c in range(D):
            assert got[i, c] == pytest.approx(kv_b[4 * (i + 1) + pick[c], c], rel=1e-12, abs=1e-12)
    last = C.compressor(x[-4:], wk[:D], wg[:D], np.zeros((4, D), np.float32), 4)
    assert np.allclose(got[G - 1], last[0], rtol=1e-12, atol=1e-12)


def pin_c4a_b_gate_selects(C):
    """The b gate, not Ape, selects: input column h0 is 1 on one chosen token
    of every group after the first and 0 elsewhere, and W^bGate has 256 in
    that column, so the chosen token's b score exceeds every other score of
    its group by about 250 and C_i = kv^b of the chosen token of group i + 1."""
    G, H, D, h0 = 4, 12, 3, 5
    x, wk, wg, ape = _rand_c4a(67, G, H, D)
    x[:, h0] = 0
    pick = [2, 0, 3]
    for i, p in enumerate(pick):
        x[4 * (i + 1) + p, h0] = bf16_bits(np.float32([1.0]))[0]
    wg[D:, h0] = bf16_bits(np.float32([256.0]))[0]
    got = C.compressor_c4a(x, wk, wg, np.zeros_like(ape))
    kv_b = _kv(x, wk[D:])
    for i, p in enumerate(pick):
        assert np.allclose(got[i], kv_b[4 * (i + 1) + p], rtol=1e-12, atol=1e-12), i


def pin_c4a_locality(C):
    """Output i depends on the rows of groups i and i + 1 only: new rows in
    group 2 move outputs 1 and 2 and no other."""
    G, H, D = 5, 8, 3
    x, wk, wg, ape = _rand_c4a(47, G, H, D)
    a = C.compressor_c4a(x, wk, wg, ape)
    x2 = x.copy()
    x2[8:12] = bf16_bits(np.random.default_rng(53).standard_normal((4, H)))
    b = C.compressor_c4a(x2, wk, wg, ape)
    for i in (0, 3, 4):
        assert np.array_equal(a[i], b[i]), i
    assert not np.allclose(a[1], b[1]) and not np.allclose(a[2], b[2])


def pin_c4a_channel_shift(C):
    """A constant per channel added to both of its Ape columns (a and b) leaves
    the outputs unchanged; added to the a column alone it moves them."""
    G, H, D = 4, 16, 3
    x, wk, wg, ape = _rand_c4a(59, G, H, D, ape_scale=2.0)
    base = C.compressor_c4a(x, wk, wg, ape)
    k = np.array([2.0, -5.0, 9.0])
    both = ape.astype(np.float64) + np.concatenate([k, k])[None, :]
    assert np.allclose(C.compressor_c4a(x, wk, wg, both), base, rtol=1e-11, atol=1e-11)
    a_only = ape.astype(np.float64) + np.concatenate([k, 0 * k])[None, :]
    assert not np.allclose(C.compressor_c4a(x, wk, wg, a_only)[:G - 1], base[:G - 1])


def pin_c4a_convexity_and_subset(C):
    """Every output channel lies within the range of the eight (last group:
    four) kv values it combines; the group-subset form returns the listed rows."""
    G, H, D = 6, 16, 4
    x, wk, wg, ape = _rand_c4a(61, G, H, D, ape_scale=3.0)
    got = C.compressor_c4a(x, wk, wg, ape)
    kv_a, kv_b = _kv(x, wk[:D]), _kv(x, wk[D:])
    for i in range(G):
        vals = np.vstack([kv_a[4 * i:4 * i + 4], kv_b[4 * i + 4:4 * i + 8]])
        assert np.all(got[i] >= vals.min(axis=0) - 1e-12) and np.all(got[i] <= vals.max(axis=0) + 1e-12)
    assert np.array_equal(C.compressor_c4a(x, wk, wg, ape, groups=[5, 0, 2]), got[[5, 0, 2]])


PINS = [pin_worked_examples, pin_group_mean, pin_row_selection, pin_row_weights_closed_form,
        pin_channel_shift_invariance, pin_permutation_equivariance, pin_group_locality, pin_convexity,
        pin_selected_groups, pin_c4a_eight_row_mean, pin_c4a_selects_an_a_row, pin_c4a_selects_a_b_row,
        pin_c4a_b_gate_selects, pin_c4a_locality, pin_c4a_channel_shift, pin_c4a_convexity_and_subset]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_compressor_oracle_pin(pin):
    pin(ORACLE)


def test_bf16_helper_is_exact():
    """The tests' own bf16 rounding: exact values survive, ties go to even."""
    vals = np.array([1.0, -2.5, 3.0, 0.0078125, 1 + 2 ** -7], dtype=np.float32)
    assert np.array_equal(exact(bf16_bits(vals)), vals.astype(np.float64))
    assert exact(bf16_bits(np.float32([1 + 2 ** -8])))[0] == 1.0              # tie -> even
    assert exact(bf16_bits(np.float32([1 + 3 * 2 ** -8])))[0] == 1 + 2 ** -6  # tie -> even (up)
