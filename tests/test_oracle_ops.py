"""Pins of the oracle's four operations (CPU only).

What pins what:
  * layout sizes      -- the pages' printed examples (kvCacheCol 323, scaleCol 4) and
                         hand-evaluated closed forms (tests/golden/layout_sizes.txt)
  * whole rows        -- hand-worked rows (tests/golden/worked_examples.txt)
  * scales            -- exact rational bounds (E8M0) and the bf16 rounding bound
  * codes             -- nearest-value search / half-spacing error bound of each format
  * skip / untouched  -- byte-identity of everything the update must not write
  * RMSNorm           -- torch.nn.functional.rms_norm in float64 (library), closed forms
  * RoPE              -- the same rotation written as complex multiplication, norm
                         preservation, identity and 90-degree special cases
  * dequant / int8    -- exact special cases and the +-0.5 rounding bound
"""
import numpy as np
import pytest
import torch

import oracle
from _formats import bf16_value, decode, nearest_code, nearest_within
from _golden import byte_pairs, expand, expand_bytes, read_cases, read_table
from _oracle_harness import row_view, run_oracle, written_mask
from kv_cache_quantize_b200 import workloads as W

WORKED = read_cases("worked_examples.txt")


def bf16_bits(vals) -> np.ndarray:
    return W.to_bf16_bits(np.asarray(vals, dtype=np.float32))


def filled_cache(num_blocks, block_size, head_dim, elem_bytes=1, inner=1, fill=0xA5):
    c = W.make_cache(np.random.default_rng(0), num_blocks, block_size, head_dim, elem_bytes, inner)
    c.storage[:] = fill
    return c


# ---------------------------------------------------------------------------
# layout sizes
# ---------------------------------------------------------------------------
def test_layout_sizes_printed_and_closed_form():
    rows = read_table("layout_sizes.txt")
    assert any(r[-1] == "printed" for r in rows)
    for r in rows:
        op, d, mode, g, expected = r[0], int(r[1]), int(r[2]), r[3], int(r[4])
        if op == "compress":
            assert oracle.kv_cache_col(d, mode, int(g)) == expected, r
        else:
            assert oracle.indexer_scale_col(d, mode) == expected, r


# ---------------------------------------------------------------------------
# hand-worked rows
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name", [k for k, v in WORKED.items() if v["op"] == "compress"])
def test_compress_worked_rows(name):
    c = WORKED[name]
    d, n = int(c["d"]), int(c["row_len"])
    xdt = c.get("x_dtype", "bf16")
    vals = expand(c["x"], d)
    x = (bf16_bits(vals) if xdt == "bf16" else np.asarray(vals, dtype=np.float16).view(np.uint16))[None, :]
    cache = filled_cache(1, 2, n + 16)
    st = cache.storage.copy()
    f = oracle.kv_compress_epilog(x, [1], oracle.Paged(st, cache.offset, 1, 2, n + 16, 2 * (n + 16)),
                                  int(c["mode"]), int(c["G"]), float(c["x_scale"]), x_dtype=xdt)
    assert f == 0
    assert oracle.kv_cache_col(d, int(c["mode"]), int(c["G"])) == n
    row = row_view(cache, st, 1, n + 16)
    assert bytes(row[:n]) == expand_bytes(c["row"], n), name
    assert np.all(row[n:] == 0xA5), "bytes past kvCacheCol must stay untouched"
    assert np.all(row_view(cache, st, 0, n + 16) == 0xA5), "slot 0 was not addressed"


@pytest.mark.parametrize("name", [k for k, v in WORKED.items() if v["op"] == "indexer"])
def test_indexer_worked_rows(name):
    c = WORKED[name]
    d, n, ns = int(c["d"]), int(c["row_len"]), int(c["scale_len"])
    x = bf16_bits(expand(c["x"], d))[None, :]
    cache = filled_cache(1, 1, n + 8)
    cs = filled_cache(1, 1, ns + 4)
    st, ss = cache.storage.copy(), cs.storage.copy()
    oracle.indexer_quant_cache(x, "bf16", [0], oracle.Paged(st, cache.offset, 1, 1, n + 8, n + 8),
                               "e4m3", oracle.Paged(ss, cs.offset, 1, 1, ns + 4, ns + 4), int(c["mode"]))
    assert bytes(row_view(cache, st, 0, n)) == expand_bytes(c["row"], n), name
    assert np.all(row_view(cache, st, 0, n + 8)[n:] == 0xA5)
    assert bytes(row_view(cs, ss, 0, ns)) == expand_bytes(c["scale"], ns), name
    assert np.all(row_view(cs, ss, 0, ns + 4)[ns:] == 0xA5)


def _rms_worked(ckv_dtype, scale):
    c = WORKED["rmsnorm_rope_d12"]
    kv = bf16_bits(expand(c["kv"], 12)).reshape(1, 1, 1, 12)
    gamma = bf16_bits(expand(c["gamma"], 8))
    cos = bf16_bits(expand(c["cos"], 4)).reshape(1, 1, 1, 4)
    sin = bf16_bits(expand(c["sin"], 4)).reshape(1, 1, 1, 4)
    eb = 2 if ckv_dtype == "bf16" else 1
    kc, cc = filled_cache(1, 2, 4, 2), filled_cache(1, 2, 8, eb)
    ks, cs = kc.storage.copy(), cc.storage.copy()
    ko = oracle.CacheOut(oracle.Paged(ks, kc.offset, 1, 2, 8, 16), "bf16")
    co = oracle.CacheOut(oracle.Paged(cs, cc.offset, 1, 2, 8 * eb, 16 * eb), ckv_dtype,
                         None if scale is None else np.array([scale], np.float32))
    f = oracle.kv_rmsnorm_rope_cache(kv, "bf16", 8, gamma, cos, sin, [1], "PA_BNSD", ko, co, 0.0)
    assert f == 0
    return c, kc, ks, cc, cs


def test_rmsnorm_rope_worked_row_e4m3():
    c, kc, ks, cc, cs = _rms_worked("e4m3", 1.0 / 64.0)
    assert bytes(row_view(cc, cs, 1, 8)) == expand_bytes(c["ckv_e4m3_row"], 8)
    assert bytes(row_view(kc, ks, 1, 8)) == expand_bytes(c["k_bf16_row"], 8)
    assert np.all(row_view(cc, cs, 0, 8) == 0xA5) and np.all(row_view(kc, ks, 0, 8) == 0xA5)


def test_rmsnorm_rope_worked_row_bf16():
    c, kc, ks, cc, cs = _rms_worked("bf16", None)
    assert bytes(row_view(cc, cs, 1, 16)) == expand_bytes(c["ckv_bf16_row"], 16)


@pytest.mark.parametrize("name", ["dequant_rope_quant_identity", "dequant_rope_quant_rot90"])
def test_dequant_rope_quant_worked_rows(name):
    c = WORKED[name]
    x = np.array(expand(c["x"], 12), dtype=np.int32).reshape(1, 1, 12)
    cos = bf16_bits(expand(c["cos"], 4)).reshape(1, 1, 1, 4)
    sin = bf16_bits(expand(c["sin"], 4)).reshape(1, 1, 1, 4)
    kc, vc = filled_cache(2, 2, 4), filled_cache(2, 2, 4)
    ks, vs = kc.storage.copy(), vc.storage.copy()
    q, k, v, f = oracle.dequant_rope_quant_kvcache(
        x, "i32", cos, sin, "bf16", oracle.Paged(ks, kc.offset, 2, 2, 4, 8), oracle.Paged(vs, vc.offset, 2, 2, 4, 8),
        [3], np.ones(4), np.full(4, 2.0), np.zeros(4), np.ones(4), np.full(12, 0.5), [2.0], np.ones(12), "f32",
        (4, 4, 4), "page", False)
    assert f == 0 and q.shape == (1, 1, 1, 4) and k is None and v is None
    assert q.view(np.uint8).tobytes() == expand_bytes(c["q_out"], 8)
    assert bytes(row_view(kc, ks, 3, 4)) == expand_bytes(c["k_row"], 4)
    assert bytes(row_view(vc, vs, 3, 4)) == expand_bytes(c["v_row"], 4)
    for s in range(3):
        assert np.all(row_view(kc, ks, s, 4) == 0xA5) and np.all(row_view(vc, vs, s, 4) == 0xA5)


# ---------------------------------------------------------------------------
# kv_compress_epilog on random data: bounds, exact scale rules, untouched bytes
# ---------------------------------------------------------------------------
def _compress_case(mode, G, kind, d=576, T=96, pad=0, slot_dtype=np.int32):
    col = oracle.kv_cache_col(d, mode, G)
    return W.gen_compress(f"c{mode}", T=T, d=d, quant_mode=mode, num_blocks=16, block_size=16,
                          head_dim=col + 13, group_size=G, x_scale=0.1, skip_frac=0.1,
                          outlier_frac=0.05, seed=3 + mode, x_kind=kind, block_pad_bytes=pad,
                          slot_dtype=slot_dtype), col


def _untouched_ok(case, st, name, nbytes, slots):
    cb = case.caches[name]
    m = written_mask(cb, slots, nbytes)
    assert np.array_equal(st[~m], cb.storage[~m]), "bytes outside the written rows changed"


@pytest.mark.parametrize("kind", ["normal", "wide"])
@pytest.mark.parametrize("mode,G", [(0, 64), (1, 64), (2, 16), (2, 32), (2, 64)])
def test_compress_random_rows_obey_the_formulas(mode, G, kind):
    case, col = _compress_case(mode, G, kind, pad=48 if mode == 1 else 0)
    sts, _, faults = run_oracle(case)
    st = sts["cache"]
    assert faults == 0
    cb = case.caches["cache"]
    slots = case.arrays["slot_mapping"]
    _untouched_ok(case, st, "cache", col, slots)
    x = case.arrays["x"]
    d, n = x.shape[1], x.shape[1] - 64
    for t in np.nonzero(slots != -1)[0]:
        row = row_view(cb, st, int(slots[t]), col)
        xv = bf16_value(x[t]).astype(np.float64)
        if mode in (0, 1):
            assert bytes(row[n:n + 128]) == x[t, n:].astype("<u2").tobytes(), "rope must be copied"
            codes = row[:n].astype(np.int64)
            for g in range(n // 64):
                xg = xv[64 * g:64 * g + 64]
                a = np.max(np.abs(xg))
                if mode == 0:
                    sb = int(row[n + 128 + 2 * g]) | (int(row[n + 129 + 2 * g]) << 8)
                    sf = float(bf16_value(sb))
                    q = a / 448.0
                    assert abs(sf - q) <= max(2.0 ** -8 * q * (1 + 2.0 ** -20), 2.0 ** -134), (t, g)
                    cg = codes[64 * g:64 * g + 64]
                    if sf == 0:
                        assert np.all(cg == 0)
                    else:
                        assert np.all(nearest_within("e4m3", xg / sf, cg)), (t, g)
                else:
                    b = int(row[n + 128 + g])
                    q = a / 448.0
                    assert 2.0 ** (b - 127) >= q and (b == 0 or 2.0 ** (b - 128) < q), (t, g)
                    r = xg * 2.0 ** (127 - b)
                    assert np.all(np.abs(r) <= 448.0)
                    assert np.array_equal(codes[64 * g:64 * g + 64], nearest_code("e4m3", r)), (t, g)
            assert np.all(row[n + 128 + (n // 64) * (2 if mode == 0 else 1):] == 0), "zero padding"
        else:
            nib = np.empty(n, dtype=np.int64)
            nib[0::2] = row[:n // 2] & 0xF
            nib[1::2] = row[:n // 2] >> 4
            for g in range(n // G):
                xg = xv[G * g:G * g + G]
                a = np.max(np.abs(xg))
                off = n // 2 + 64 + 2 * g
                sf = float(bf16_value(int(row[off]) | (int(row[off + 1]) << 8)))
                q = a / 6.0
                assert abs(sf - q) <= max(2.0 ** -8 * q * (1 + 2.0 ** -20), 2.0 ** -134), (t, g)
                if sf == 0:
                    assert np.all(nib[G * g:G * g + G] == 0)
                else:
                    assert np.all(nearest_within("e2m1", xg / sf, nib[G * g:G * g + G])), (t, g)
            rope = row[n // 2:n // 2 + 64]
            xs = float(np.float32(0.1))
            assert np.all(nearest_within("e4m3", xv[n:] * xs, rope)), t
            assert np.all(row[n // 2 + 64 + 2 * (n // G):] == 0), "zero padding"


@pytest.mark.parametrize("mode,G", [(0, 64), (1, 64), (2, 32)])
def test_compress_tiny_rows_brute_force(mode, G):
    """Tiny rows: codes from an exhaustive nearest search of the binary32 quotient."""
    d, T = 128, 6
    case = W.gen_compress("tiny", T=T, d=d, quant_mode=mode, num_blocks=1, block_size=T,
                          head_dim=oracle.kv_cache_col(d, mode, G), group_size=G, x_scale=0.5,
                          seed=17, x_kind="wide")
    case.arrays["slot_mapping"] = np.arange(T, dtype=np.int32)
    st, _, _ = run_oracle(case)
    col = oracle.kv_cache_col(d, mode, G)
    for t in range(T):
        row = row_view(case.caches["cache"], st["cache"], t, col)
        x32 = bf16_value(case.arrays["x"][t])
        n = d - 64
        gs = 64 if mode < 2 else G
        for g in range(n // gs):
            xg = x32[gs * g:gs * (g + 1)]
            a = np.float32(np.max(np.abs(xg)))
            if mode == 1:
                b = int(row[n + 128 + g])
                v = xg * np.float32(2.0 ** (127 - b))
                assert np.array_equal(row[gs * g:gs * (g + 1)], nearest_code("e4m3", v))
                continue
            fmax = np.float32(448.0 if mode == 0 else 6.0)
            sb = W.to_bf16_bits(np.array([a / fmax], np.float32))[0]
            sf = bf16_value(sb)
            want = np.zeros(gs, np.uint32) if sf == 0 else nearest_code(
                "e4m3" if mode == 0 else "e2m1", (xg / sf).astype(np.float32))
            if mode == 0:
                got = row[gs * g:gs * (g + 1)]
            else:
                nb = row[(gs * g) // 2:(gs * (g + 1)) // 2]
                got = np.empty(gs, np.int64)
                got[0::2], got[1::2] = nb & 0xF, nb >> 4
            assert np.array_equal(got, want), (t, g)


def test_compress_skips_minus_one_and_flags_out_of_range():
    case, col = _compress_case(0, 64, "normal", T=40)
    s = case.arrays["slot_mapping"]
    s[:5] = -1
    s[5] = case.caches["cache"].num_slots      # one past the end
    s[6] = -7
    sts, _, faults = run_oracle(case)
    assert faults == oracle.FAULT_SLOT_RANGE
    _untouched_ok(case, sts["cache"], "cache", col, s)
    all_skipped = case.arrays["slot_mapping"].copy()
    all_skipped[:] = -1
    case.arrays["slot_mapping"] = all_skipped
    st2, _, f2 = run_oracle(case)
    assert f2 == 0 and np.array_equal(st2["cache"], case.caches["cache"].storage)


def test_compress_int64_slots_give_the_same_bytes():
    a, col = _compress_case(2, 32, "normal", slot_dtype=np.int32)
    b, _ = _compress_case(2, 32, "normal", slot_dtype=np.int64)
    assert np.array_equal(run_oracle(a)[0]["cache"], run_oracle(b)[0]["cache"])


# ---------------------------------------------------------------------------
# indexer_quant_cache
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("x_dtype", ["bf16", "f16"])
@pytest.mark.parametrize("mode,cdt,d", [(0, "e4m3", 128), (0, "e5m2", 100), (3, "u8", 128), (3, "u8", 99),
                                        (1, "e4m3", 128), (1, "e5m2", 64)])
def test_indexer_random_rows_obey_the_formulas(mode, cdt, d, x_dtype):
    scol = oracle.indexer_scale_col(d, mode)
    code_bytes = (d + 1) // 2 if mode == 3 else d
    sbytes = 4 if mode == 1 else scol
    case = W.gen_indexer("i", T=80, d=d, quant_mode=mode, num_blocks=32, block_size=4,
                         cache_head_dim=code_bytes + 5, scale_head_dim=scol + 3, cache_dtype=cdt,
                         x_dtype=x_dtype, skip_frac=0.1, seed=5, block_pad_bytes=32)
    st, _, f = run_oracle(case)
    assert f == 0
    slots = case.arrays["slot_mapping"]
    for nm, nb in (("cache", code_bytes), ("cache_scale", sbytes)):
        m = written_mask(case.caches[nm], slots, nb)
        assert np.array_equal(st[nm][~m], case.caches[nm].storage[~m]), nm
    fmt = "e5m2" if cdt == "e5m2" else "e4m3"
    fp_max = 57344.0 if cdt == "e5m2" else 448.0
    x = case.arrays["x"]
    xv_all = (bf16_value(x) if x_dtype == "bf16" else x.view(np.float16).astype(np.float32)).astype(np.float64)
    for t in np.nonzero(slots != -1)[0]:
        s = int(slots[t])
        row = row_view(case.caches["cache"], st["cache"], s, code_bytes).astype(np.int64)
        srow = row_view(case.caches["cache_scale"], st["cache_scale"], s, sbytes)
        xv = xv_all[t]
        if mode == 1:
            scale = float(srow.view(np.float32)[0])
            a = np.max(np.abs(xv))
            assert abs(scale - a / fp_max) <= 2.0 ** -24 * a / fp_max
            if scale == 0:
                assert np.all(row == 0)
            else:
                assert np.all(nearest_within(fmt, xv / scale, row))
            continue
        if mode == 3:
            codes = np.empty(2 * code_bytes, np.int64)
            codes[0::2], codes[1::2] = row & 0xF, row >> 4
            if d % 2:
                assert codes[-1] == 0
            codes = codes[:d]
        else:
            codes = row
        fm = 6.0 if mode == 3 else fp_max
        for g in range(scol):
            xg = xv[32 * g:32 * g + 32]
            b = int(srow[g])
            q = np.max(np.abs(xg)) / fm
            assert 2.0 ** (b - 127) >= q and (b == 0 or 2.0 ** (b - 128) < q)
            r = xg * 2.0 ** (127 - b)
            assert np.all(np.abs(r) <= fm)
            assert np.array_equal(codes[32 * g:32 * g + 32], nearest_code("e2m1" if mode == 3 else fmt, r))


# ---------------------------------------------------------------------------
# kv_rmsnorm_rope_cache
# ---------------------------------------------------------------------------
def _rms_case(k_dtype="bf16", ckv_dtype="bf16", cache_mode="PA_BNSD", B=12, S=1, ckv_scale=None,
              ckv_offset=None, k_scale=None, seed=7):
    return W.gen_rmsnorm_rope("r", B=B, S=S, D=576, Dv=512, num_blocks=8, block_size=16, k_dtype=k_dtype,
                              ckv_dtype=ckv_dtype, ckv_scale=ckv_scale, ckv_offset=ckv_offset, k_scale=k_scale,
                              cache_mode=cache_mode, skip_frac=0.1, seed=seed, block_pad_bytes=64)


def _token_slots(case):
    """(token index, slot) pairs per the index semantics of each cache mode."""
    at, idx = case.attrs, case.arrays["index"].astype(np.int64)
    B, S = case.arrays["kv"].shape[0], case.arrays["kv"].shape[2]
    bs = case.caches["k_cache"].block_size
    out = []
    for b in range(B):
        for s in range(S):
            t = b * S + s
            if at["cache_mode"] == "Norm":
                v = idx.reshape(B, S)[b, s]
                slot = -1 if v == -1 else b * bs + v
            elif at["cache_mode"] == "PA_BLK_BNSD":
                nb = (S + bs - 1) // bs
                v = idx[b * nb + s // bs]
                slot = -1 if v == -1 else (v // bs) * bs + s % bs
            else:
                slot = idx[t]
            if slot != -1:
                out.append((t, int(slot)))
    return out


def _rms_reference(case):
    """float64 RMSNorm through torch.nn.functional.rms_norm and the rotation as a complex product."""
    kv = bf16_value(case.arrays["kv"]).astype(np.float64).reshape(-1, 576)
    gamma = bf16_value(case.arrays["gamma"]).astype(np.float64)
    y = torch.nn.functional.rms_norm(torch.from_numpy(kv[:, :512]), [512], torch.from_numpy(gamma),
                                     eps=case.attrs["epsilon"]).numpy()
    cos = bf16_value(case.arrays["cos"]).astype(np.float64).reshape(-1, 64)
    sin = bf16_value(case.arrays["sin"]).astype(np.float64).reshape(-1, 64)
    z = kv[:, 512:]
    zc = (z[:, 0::2] + 1j * z[:, 1::2]) * (cos[:, :32] + 1j * sin[:, :32])   # cos/sin halves are equal
    rope = np.concatenate([zc.real, zc.imag], axis=1)
    return y, rope


@pytest.mark.parametrize("cache_mode", ["PA_BNSD", "PA", "Norm", "PA_BLK_BNSD"])
def test_rmsnorm_rope_matches_float64_textbook(cache_mode):
    S = 1 if cache_mode in ("PA_BNSD", "PA") else 5
    case = _rms_case(cache_mode=cache_mode, B=6 if S > 1 else 12, S=S)
    st, _, f = run_oracle(case)
    assert f == 0
    y, rope = _rms_reference(case)
    pairs = _token_slots(case)
    assert pairs, "some tokens must be written"
    for nm, nb in (("ckv_cache", 1024), ("k_cache", 128)):
        m = written_mask(case.caches[nm], [s for _, s in pairs], nb)
        assert np.array_equal(st[nm][~m], case.caches[nm].storage[~m]), nm
    for t, s in pairs:
        ckv = bf16_value(row_view(case.caches["ckv_cache"], st["ckv_cache"], s, 1024).view(np.uint16))
        k = bf16_value(row_view(case.caches["k_cache"], st["k_cache"], s, 128).view(np.uint16))
        np.testing.assert_allclose(ckv, y[t], rtol=1e-2, atol=1e-6)
        np.testing.assert_allclose(k, rope[t], rtol=1e-2, atol=1e-5)


def test_rmsnorm_invariants_and_constant_row():
    case = _rms_case()
    st, _, _ = run_oracle(case)
    kv = bf16_value(case.arrays["kv"]).astype(np.float64).reshape(-1, 576)
    gamma = bf16_value(case.arrays["gamma"]).astype(np.float64)
    for t, s in _token_slots(case):
        y = bf16_value(row_view(case.caches["ckv_cache"], st["ckv_cache"], s, 1024).view(np.uint16))
        ms = np.mean(kv[t, :512] ** 2)
        np.testing.assert_allclose(np.mean((y / gamma) ** 2), ms / (ms + 1e-6), rtol=1e-2)
        # norm of every rotated pair is preserved
        k = bf16_value(row_view(case.caches["k_cache"], st["k_cache"], s, 128).view(np.uint16)).astype(np.float64)
        z = kv[t, 512:]
        np.testing.assert_allclose(k[:32] ** 2 + k[32:] ** 2, z[0::2] ** 2 + z[1::2] ** 2, rtol=2e-2, atol=1e-4)
    # gamma = 1 and a constant row c: y = c / sqrt(c^2 + eps) everywhere
    c0 = 0.75
    case.arrays["kv"][:] = W.to_bf16_bits(np.full(case.arrays["kv"].shape, c0, np.float32))
    case.arrays["gamma"][:] = W.to_bf16_bits(np.ones(512, np.float32))
    st, _, _ = run_oracle(case)
    want = c0 / np.sqrt(c0 * c0 + 1e-6)
    for _, s in _token_slots(case):
        y = bf16_value(row_view(case.caches["ckv_cache"], st["ckv_cache"], s, 1024).view(np.uint16))
        np.testing.assert_allclose(y, want, rtol=4e-3)


def test_rope_identity_and_quarter_turn_are_exact():
    case = _rms_case()
    shape = case.arrays["cos"].shape
    z = bf16_value(case.arrays["kv"]).reshape(-1, 576)[:, 512:]
    for c0, s0, want in ((1.0, 0.0, np.concatenate([z[:, 0::2], z[:, 1::2]], 1)),
                         (0.0, 1.0, np.concatenate([-z[:, 1::2], z[:, 0::2]], 1))):
        case.arrays["cos"] = W.to_bf16_bits(np.full(shape, c0, np.float32))
        case.arrays["sin"] = W.to_bf16_bits(np.full(shape, s0, np.float32))
        st, _, _ = run_oracle(case)
        for t, s in _token_slots(case):
            k = bf16_value(row_view(case.caches["k_cache"], st["k_cache"], s, 128).view(np.uint16))
            assert np.array_equal(k, want[t].astype(np.float32))


@pytest.mark.parametrize("ckv_dtype,scale,offset", [("e4m3", 1 / 64, None), ("e5m2", 1 / 64, None),
                                                    ("i8", 1 / 32, 3.0)])
def test_rmsnorm_quantised_ckv_within_format_bound(ckv_dtype, scale, offset):
    case = _rms_case(ckv_dtype=ckv_dtype, ckv_scale=[scale], ckv_offset=None if offset is None else [offset])
    st, _, _ = run_oracle(case)
    y, _ = _rms_reference(case)
    for t, s in _token_slots(case):
        row = row_view(case.caches["ckv_cache"], st["ckv_cache"], s, 512)
        r = y[t] / scale
        if ckv_dtype == "i8":
            v = row.view(np.int8).astype(np.float64)
            target = np.clip(r + offset, -128, 127)
            assert np.all(np.abs(v - target) <= 0.5 + 1e-2 * np.abs(r) + 1e-3)
        else:
            # the binary32 y differs from the float64 one by ~1e-6 relative: allow it as slack
            assert np.all(nearest_within(ckv_dtype, r, row, slack_rel=2e-5))


def test_rmsnorm_quantised_k_cache():
    case = _rms_case(k_dtype="e4m3", ckv_dtype="bf16", k_scale=[1 / 16])
    st, _, _ = run_oracle(case)
    _, rope = _rms_reference(case)
    for t, s in _token_slots(case):
        row = row_view(case.caches["k_cache"], st["k_cache"], s, 64)
        assert np.all(nearest_within("e4m3", rope[t] * 16, row, slack_rel=2e-5))


# ---------------------------------------------------------------------------
# dequant_rope_quant_kvcache
# ---------------------------------------------------------------------------
def _drq_case(**kw):
    base = dict(B=3, S=8, Nq=4, Nkv=2, D=64, c0=6, c1=8, x_range=1 << 12, seed=9, block_pad_bytes=40)
    base.update(kw)
    return W.gen_dequant_rope_quant("d", **base)


def _drq_reference(case):
    a, at = case.arrays, case.attrs
    x = a["x"].astype(np.float64)
    B = x.shape[0]
    H = x.shape[-1]
    x = x.reshape(-1, H)
    v = x * a["weight_scale"].astype(np.float64)
    if "activation_scale" in a:
        v = v * a["activation_scale"].astype(np.float64)[:, None]
    if "bias" in a:
        v = v + a["bias"].astype(np.float64)
    D, Nq, Nkv = at["D"], at["Nq"], at["Nkv"]
    cos = bf16_value(a["cos"]).astype(np.float64).reshape(-1, D)
    sin = bf16_value(a["sin"]).astype(np.float64).reshape(-1, D)
    h = D // 2
    heads = v[:, :(Nq + Nkv) * D].reshape(-1, Nq + Nkv, D)
    u = heads[..., :h] + 1j * heads[..., h:]
    rot = u * (cos[:, None, :h] + 1j * sin[:, None, :h])
    o = np.concatenate([rot.real, rot.imag], axis=-1)
    return o[:, :Nq], o[:, Nq:], v[:, (Nq + Nkv) * D:].reshape(-1, Nkv, D), B


@pytest.mark.parametrize("cache_mode", ["page", "contiguous"])
def test_dequant_rope_quant_matches_float64_rotation(cache_mode):
    case = _drq_case(cache_mode=cache_mode, kv_output=True, skip_frac=0.1 if cache_mode == "page" else 0.0)
    st, outs, f = run_oracle(case)
    assert f == 0
    q_ref, k_ref, v_ref, B = _drq_reference(case)
    at, a = case.attrs, case.arrays
    S = a["x"].shape[1]
    q = bf16_value(outs["q_out"]).reshape(q_ref.shape)
    np.testing.assert_allclose(q, q_ref, rtol=1e-2, atol=1e-4)
    np.testing.assert_allclose(bf16_value(outs["k_out"]).reshape(k_ref.shape), k_ref, rtol=1e-2, atol=1e-4)
    np.testing.assert_allclose(bf16_value(outs["v_out"]).reshape(v_ref.shape), v_ref, rtol=1e-2, atol=1e-4)
    sk = a["scale_k"].reshape(-1).astype(np.float64)
    sv = a["scale_v"].reshape(-1).astype(np.float64)
    ok_, ov_ = a["offset_k"].reshape(-1), a["offset_v"].reshape(-1)
    kc, vc = case.caches["k_cache"], case.caches["v_cache"]
    nb = kc.row_bytes
    written = []
    for t in range(B * S):
        b, s = divmod(t, S)
        if cache_mode == "page":
            slot = int(a["indices"][t])
            if slot == -1:
                continue
        else:
            slot = b * kc.block_size + int(a["indices"][b]) + s
        written.append(slot)
        kq = row_view(kc, st["k_cache"], slot, nb).view(np.int8).astype(np.float64)
        vq = row_view(vc, st["v_cache"], slot, nb).view(np.int8).astype(np.float64)
        for got, ref, sc, of in ((kq, k_ref[t].reshape(-1), sk, ok_), (vq, v_ref[t].reshape(-1), sv, ov_)):
            target = ref / sc + of
            clipped = np.clip(target, -128, 127)
            assert np.all(np.abs(got - clipped) <= 0.5 + 1e-4 * np.abs(target) + 1e-3)
    for nm in ("k_cache", "v_cache"):
        m = written_mask(case.caches[nm], written, nb)
        assert np.array_equal(st[nm][~m], case.caches[nm].storage[~m]), nm


def test_dequant_special_case_is_exact():
    case = _drq_case(with_offsets=False, with_activation_scale=False, bias_dtype=None, x_range=100)
    a = case.arrays
    a["weight_scale"][:] = 1.0
    a["scale_k"][:] = 1.0
    a["scale_v"][:] = 1.0
    a["cos"][:] = W.to_bf16_bits(np.ones(1, np.float32))[0]
    a["sin"][:] = W.to_bf16_bits(np.zeros(1, np.float32))[0]
    st, outs, _ = run_oracle(case)
    at = case.attrs
    D, Nq, Nkv = at["D"], at["Nq"], at["Nkv"]
    x = a["x"].reshape(-1, (Nq + 2 * Nkv) * D)
    assert np.array_equal(bf16_value(outs["q_out"]).reshape(-1, Nq * D), x[:, :Nq * D].astype(np.float32))
    kc = case.caches["k_cache"]
    for t in range(x.shape[0]):
        slot = int(a["indices"][t])
        if slot == -1:
            continue
        k = row_view(kc, st["k_cache"], slot, kc.row_bytes).view(np.int8)
        assert np.array_equal(k, np.clip(x[t, Nq * D:(Nq + Nkv) * D], -128, 127).astype(np.int8))


def test_dequant_two_dim_x_and_shapes():
    case = _drq_case(S=1, x_2d=True, kv_output=True, cache_mode="contiguous", c1=4)
    st, outs, f = run_oracle(case)
    at = case.attrs
    assert outs["q_out"].shape == (3, at["Nq"], at["D"])
    assert outs["k_out"].shape == (3, at["Nkv"], at["D"]) == outs["v_out"].shape
    none = _drq_case(kv_output=False)
    _, o2, _ = run_oracle(none)
    assert o2["k_out"] is None and o2["v_out"] is None


@pytest.mark.parametrize("bias_dtype", ["f32", "bf16", "f16", "i32"])
def test_dequant_bias_dtypes(bias_dtype):
    case = _drq_case(bias_dtype=bias_dtype)
    st, outs, f = run_oracle(case)
    a = case.arrays
    if bias_dtype in ("bf16", "f16"):
        bias = (bf16_value(a["bias"]) if bias_dtype == "bf16" else a["bias"].view(np.float16)).astype(np.float64)
        a = dict(a)
        a["bias"] = bias
        case.arrays = a
    q_ref, _, _, _ = _drq_reference(case)
    np.testing.assert_allclose(bf16_value(outs["q_out"]).reshape(q_ref.shape), q_ref, rtol=1e-2, atol=1e-4)


def test_dequant_out_of_range_index_is_flagged():
    case = _drq_case()
    case.arrays["indices"][0] = case.caches["k_cache"].num_slots
    _, _, f = run_oracle(case)
    assert f == oracle.FAULT_SLOT_RANGE


def test_rmsnorm_epsilon_enters_under_the_square_root():
    # with eps comparable to mean(x^2) a dropped or misplaced eps moves y by tens of percent
    case = _rms_case()
    case.attrs["epsilon"] = 0.75
    st, _, _ = run_oracle(case)
    y, _ = _rms_reference(case)
    for t, s in _token_slots(case):
        ckv = bf16_value(row_view(case.caches["ckv_cache"], st["ckv_cache"], s, 1024).view(np.uint16))
        np.testing.assert_allclose(ckv, y[t], rtol=1e-2, atol=1e-6)


def _random_tables(shape, seed):
    r = np.random.default_rng(seed)
    return (W.to_bf16_bits(r.uniform(-1, 1, shape).astype(np.float32)),
            W.to_bf16_bits(r.uniform(-1, 1, shape).astype(np.float32)))


def test_interleaved_rope_with_unequal_cos_sin_halves():
    """cos/sin whose two halves differ: compare with the page's whole-vector formula
    y = cat(x1, x2) * cos + cat(-x2, x1) * sin evaluated in float64."""
    case = _rms_case()
    case.arrays["cos"], case.arrays["sin"] = _random_tables(case.arrays["cos"].shape, 71)
    st, _, _ = run_oracle(case)
    z = bf16_value(case.arrays["kv"]).astype(np.float64).reshape(-1, 576)[:, 512:]
    c = bf16_value(case.arrays["cos"]).astype(np.float64).reshape(-1, 64)
    s = bf16_value(case.arrays["sin"]).astype(np.float64).reshape(-1, 64)
    x1, x2 = z[:, 0::2], z[:, 1::2]
    want = np.concatenate([x1, x2], 1) * c + np.concatenate([-x2, x1], 1) * s
    for t, slot in _token_slots(case):
        k = bf16_value(row_view(case.caches["k_cache"], st["k_cache"], slot, 128).view(np.uint16))
        np.testing.assert_allclose(k, want[t], rtol=1e-2, atol=1e-5)


def test_half_rotation_rope_with_unequal_cos_sin_halves():
    """x * cos + rotate_half(x) * sin with rotate_half(x) = cat(-x[h:], x[:h]), float64."""
    case = _drq_case(kv_output=True)
    case.arrays["cos"], case.arrays["sin"] = _random_tables(case.arrays["cos"].shape, 72)
    _, outs, _ = run_oracle(case)
    at, a = case.attrs, case.arrays
    D, Nq, Nkv, h = at["D"], at["Nq"], at["Nkv"], at["D"] // 2
    x = a["x"].astype(np.float64).reshape(-1, (Nq + 2 * Nkv) * D)
    v = (x * a["weight_scale"] * a["activation_scale"][:, None] + a["bias"]).reshape(-1, Nq + 2 * Nkv, D)
    c = bf16_value(a["cos"]).astype(np.float64).reshape(-1, 1, D)
    s = bf16_value(a["sin"]).astype(np.float64).reshape(-1, 1, D)
    u = v[:, :Nq + Nkv]
    want = u * c + np.concatenate([-u[..., h:], u[..., :h]], -1) * s
    np.testing.assert_allclose(bf16_value(outs["q_out"]).reshape(-1, Nq, D), want[:, :Nq], rtol=1e-2, atol=1e-4)
    np.testing.assert_allclose(bf16_value(outs["k_out"]).reshape(-1, Nkv, D), want[:, Nq:], rtol=1e-2, atol=1e-4)


@pytest.mark.parametrize("mode", [0, 1])
def test_compress_f16_rope_bytes_are_the_input_bytes(mode):
    """aclnnKvCompressEpilog keeps the rope segment unchanged: with float16 x (allowed in
    quantMode 0 and 1) the rope bytes of every written row are x's own 16-bit values."""
    T, d = 40, 320
    rng = np.random.default_rng(mode)
    x = (rng.standard_normal((T, d)) * 3).astype(np.float16).view(np.uint16)
    col = oracle.kv_cache_col(d, mode, 64)
    cache = filled_cache(8, 8, col + 3)
    st = cache.storage.copy()
    slots = rng.choice(64, T, replace=False).astype(np.int32)
    slots[::7] = -1
    assert oracle.kv_compress_epilog(x, slots, oracle.Paged(st, cache.offset, 8, 8, col + 3, 8 * (col + 3)), mode,
                                     64, 1.0, x_dtype="f16") == 0
    n = d - 64
    for t, s in enumerate(slots.tolist()):
        if s < 0:
            continue
        row = row_view(cache, st, s, col)
        assert bytes(row[n:n + 128]) == x[t, n:].tobytes()


def test_compress_f16_is_refused_in_mode_2():
    """quantMode 2 needs bfloat16 x (aclnnKvCompressEpilog, 约束说明)."""
    cache = filled_cache(1, 2, 352)
    x = np.zeros((1, 576), dtype=np.uint16)
    with pytest.raises(Exception):
        oracle.kv_compress_epilog(x, [0], oracle.Paged(cache.storage.copy(), cache.offset, 1, 2, 352, 704), 2, 32,
                                  0.1, x_dtype="f16")
