"""The tcgen05 Compressor kernel against the float64 oracle (aclnnCompressor,
计算公式 steps 1-5, C128A and C4A forms), through the C ABI.

The kernel multiplies bf16 inputs on the tensor cores with fp32 accumulation
and runs the softmax in fp32, so the comparison is within a bound derived
from that arithmetic, per output (group g, channel c):

  |gpu - ref| <= 2^-8 |ref|                     one bf16 rounding of the output (half an ulp is 2^-9)
               + E_kv + 2 E_s R                 fp32 accumulation of kv_state / score_state: at most
                                                H / 16 roundings (one per 16-deep MMA step) of a partial
                                                sum bounded by A = sum_k |x_k w_k|, E = (H / 16) 2^-23 A,
                                                taken at the group's largest A; an error e in the scores
                                                moves the softmax-weighted mean by at most 2 e R with
                                                R = max_r |kv_r - ref|
               + 2^-18 M                        the approximate exponential (relative error below 2^-21
                                                per weight) and fp32 sums of <= 128 weights, M = max |kv_r|

For the C4A form the same bound is taken over a group's eight rows (its own
four tokens through the a weights, the next four through the b weights; four
for the last group).

Full-size workloads are checked on sampled groups (the first, the last and a
spread between), which the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import kv_cache_quantize_b200 as kvq
import oracle.compressor as OC
from kv_cache_quantize_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _bound(case, groups, ref):
    a = case.arrays
    ratio = case.attrs["ratio"]
    H = a["x"].shape[1]
    akv, ag = OC.abs_states(a["x"], a["w_kv"], a["w_gate"], groups, ratio)
    rows = np.concatenate([np.arange(g * ratio, (g + 1) * ratio) for g in groups])
    kv, sc = OC.states(a["x"][rows], a["w_kv"], a["w_gate"])
    G, D = len(groups), a["w_kv"].shape[0]
    kv = kv.reshape(G, ratio, D)
    sp = sc.reshape(G, ratio, D) + a["ape"].astype(np.float64)[None]
    e_kv = (H / 16) * 2.0 ** -23 * akv.reshape(G, ratio, D).max(axis=1)
    # accumulation of score_state, then one fp32 rounding of score + Ape
    e_s = (H / 16) * 2.0 ** -23 * ag.reshape(G, ratio, D).max(axis=1) + 2.0 ** -24 * np.abs(sp).max(axis=1)
    R = np.abs(kv - ref[:, None, :]).max(axis=1)
    M = np.abs(kv).max(axis=1)
    return 2.0 ** -8 * np.abs(ref) + e_kv + 2 * e_s * R + 2.0 ** -18 * M


def _check(case, groups=None):
    call, _, outs = W.build_call(case)
    kvq.get_error()
    call()
    torch.cuda.synchronize()
    assert kvq.get_error() == 0
    got = outs["cmp_kv"].float().cpu().numpy().astype(np.float64)
    ratio = case.attrs["ratio"]
    G = case.arrays["x"].shape[0] // ratio
    groups = list(range(G)) if groups is None else list(groups)
    ref = OC.compressor(case.arrays["x"], case.arrays["w_kv"], case.arrays["w_gate"], case.arrays["ape"], ratio,
                        groups=groups)
    got = got[groups]
    err = np.abs(got - ref)
    bound = _bound(case, groups, ref)
    bad = np.argwhere(err > bound)
    rel = err / np.maximum(np.abs(ref), 1e-30)
    print(f"{case.name}: max |err| {err.max():.3e}, median rel {np.median(rel):.3e}, "
          f"max err/bound {float((err / bound).max()):.3f}")
    assert bad.size == 0, (f"{case.name}: {len(bad)} outputs beyond the bound, first (group, channel) "
                           f"{tuple(bad[0])}: gpu {got[tuple(bad[0])]} ref {ref[tuple(bad[0])]}")
    return got


# ---------------------------------------------------------------------------
# C4A / C4Li (coff = 2, cmp_ratio = 4)
# ---------------------------------------------------------------------------
def _bound_c4a(case, groups, ref):
    a = case.arrays
    x, wk, wg = a["x"], a["w_kv"], a["w_gate"]
    T, H = x.shape
    D = wk.shape[0] // 2
    ape = a["ape"].astype(np.float64)
    out = []
    for n, i in enumerate(groups):
        parts = [(np.arange(4 * i, 4 * i + 4), slice(0, D)), (np.arange(4 * i + 4, min(4 * i + 8, T)), slice(D, 2 * D))]
        kv, sc, akv, ag = [], [], [], []
        for rows, half in parts:
            if len(rows) == 0:
                continue
            k_, s_ = OC.states(x[rows], wk[half], wg[half])
            X = np.abs(OC.bf16_to_f64(x[rows]))
            kv.append(k_)
            sc.append(s_ + ape[:len(rows), half])
            akv.append(X @ np.abs(OC.bf16_to_f64(wk[half])).T)
            ag.append(X @ np.abs(OC.bf16_to_f64(wg[half])).T)
        kv, sc, akv, ag = (np.vstack(v) for v in (kv, sc, akv, ag))
        e_kv = (H / 16) * 2.0 ** -23 * akv.max(axis=0)
        e_s = (H / 16) * 2.0 ** -23 * ag.max(axis=0) + 2.0 ** -24 * np.abs(sc).max(axis=0)
        R = np.abs(kv - ref[n][None, :]).max(axis=0)
        M = np.abs(kv).max(axis=0)
        out.append(2.0 ** -8 * np.abs(ref[n]) + e_kv + 2 * e_s * R + 2.0 ** -18 * M)
    return np.array(out)


def _check_c4a(case, groups=None):
    call, _, outs = W.build_call(case)
    kvq.get_error()
    call()
    torch.cuda.synchronize()
    assert kvq.get_error() == 0
    got = outs["cmp_kv"].float().cpu().numpy().astype(np.float64)
    G = case.arrays["x"].shape[0] // 4
    groups = list(range(G)) if groups is None else list(groups)
    a = case.arrays
    ref = OC.compressor_c4a(a["x"], a["w_kv"], a["w_gate"], a["ape"], groups=groups)
    got = got[groups]
    err = np.abs(got - ref)
    bound = _bound_c4a(case, groups, ref)
    bad = np.argwhere(err > bound)
    print(f"{case.name}: max |err| {err.max():.3e}, max err/bound {float((err / bound).max()):.3f}")
    assert bad.size == 0, (f"{case.name}: {len(bad)} outputs beyond the bound, first (group, channel) "
                           f"{tuple(bad[0])}: gpu {got[tuple(bad[0])]} ref {ref[tuple(bad[0])]}")
    return got


@pytest.mark.parametrize("T", [4, 8, 400, 2048, 5120])
def test_compressor_c4a(T):
    """D 512: one group (no next tokens at all), two groups, a ragged last tile,
    128-token tiles (T 2048: 17 tiles of 31 groups per channel tile) and
    256-token tiles (T 5120: 21 tiles of 63 groups)."""
    _check_c4a(W.gen_compressor(f"c4a_T{T}", T=T, H=1024, D=512, ratio=4, seed=T, coff=2))


@pytest.mark.parametrize("T", [2048, 20480])
def test_compressor_c4li(T):
    """D 128 (C4Li): 128- and 256-token tiles."""
    _check_c4a(W.gen_compressor(f"c4li_T{T}", T=T, H=1536, D=128, ratio=4, seed=T + 1, coff=2))


@pytest.mark.parametrize("H", [1536, 10240])
def test_compressor_c4a_hidden_sizes(H):
    _check_c4a(W.gen_compressor(f"c4a_H{H}", T=512, H=H, D=512, ratio=4, seed=H, coff=2, ape_scale=3.0))


def test_compressor_c4a_selects_rows():
    """Dominant Ape entries in the a columns for half of the channels and in the
    b columns for the other half: every output equals one kv value of the own
    four tokens (a) or of the next four (b), which pins the pairing of the a
    and b rows and the window of the b part on the device, up to the output
    rounding."""
    case = W.gen_compressor("c4a_select", T=1024, H=1024, D=128, ratio=4, seed=5, coff=2)
    D = 128
    rng = np.random.default_rng(11)
    pick = rng.integers(0, 4, D)
    ape = np.zeros((4, 2 * D), np.float32)
    ape[pick[:64], np.arange(64)] = 80.0
    ape[pick[64:], D + np.arange(64, 128)] = 80.0
    case.arrays["ape"] = ape
    _check_c4a(case)


def test_compressor_c4a_full_size_sampled_groups():
    case = W.compressor_c4a_T65536_H7168_D512()
    G = case.arrays["x"].shape[0] // 4
    # the first and last groups, tile edges of the 256-token tiles (63 groups each) and a spread
    _check_c4a(case, groups=[0, 1, 62, 63, 64, 125, 126, 127, 4000, 9999, G - 64, G - 63, G - 2, G - 1])


def test_compressor_c4a_small_named_workload():
    _check_c4a(W.compressor_c4a_T2048_H1024_D512())


@pytest.mark.parametrize("D", [128, 512])
@pytest.mark.parametrize("ratio", [2, 4, 8, 16, 32, 64, 128])
def test_compressor_ratios(ratio, D):
    """768 rows (six 128-token tiles), every ratio, both channel counts."""
    _check(W.gen_compressor(f"cp_r{ratio}_D{D}", T=768, H=1024, D=D, ratio=ratio, seed=ratio + D))


@pytest.mark.parametrize("ratio", [2, 32, 128])
def test_compressor_wide_token_tiles(ratio):
    """A batch large enough for 256-token tiles (T 5120, D 512: 80 tiles);
    the cases above, at most 74 tiles of 256, run 128-token tiles."""
    _check(W.gen_compressor(f"cp_wide_r{ratio}", T=5120, H=1024, D=512, ratio=ratio, seed=7 + ratio))


def test_compressor_wide_token_tiles_d128():
    _check(W.gen_compressor("cp_wide_d128", T=19200, H=1024, D=128, ratio=64, seed=11))


@pytest.mark.parametrize("T", [128, 384, 2176])
def test_compressor_ragged_token_tiles(T):
    """T not a multiple of the token tile: the last tile holds one group."""
    _check(W.gen_compressor(f"cp_T{T}", T=T, H=2048, D=512, ratio=128, seed=T))


@pytest.mark.parametrize("H", [1536, 4096, 10240])
def test_compressor_hidden_sizes(H):
    _check(W.gen_compressor(f"cp_H{H}", T=512, H=H, D=512, ratio=128, seed=H, ape_scale=3.0))


def test_compressor_small_named_workload():
    _check(W.compressor_c128a_T2048_H1024_D512())


def test_compressor_full_size_sampled_groups():
    case = W.compressor_c128a_T65536_H7168_D512()
    G = case.arrays["x"].shape[0] // 128
    _check(case, groups=[0, 1, 2, 3, 127, 128, 255, 256, 300, 411, G - 2, G - 1])


def test_compressor_deterministic_and_repeatable():
    case = W.compressor_c128a_T2048_H1024_D512(seed=3)
    call, _, outs = W.build_call(case)
    call()
    torch.cuda.synchronize()
    first = outs["cmp_kv"].clone()
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    assert torch.equal(first, outs["cmp_kv"])


def test_compressor_large_scores_select_rows():
    """A dominant Ape entry per channel selects one row of kv_state (the page's
    softmax over the group's rows), which the kernel must reproduce exactly up
    to the output rounding."""
    case = W.gen_compressor("cp_select", T=512, H=1024, D=128, ratio=128, seed=5)
    pick = np.random.default_rng(9).integers(0, 128, 128)
    ape = np.zeros((128, 128), np.float32)
    ape[pick, np.arange(128)] = 80.0
    case.arrays["ape"] = ape
    _check(case)
