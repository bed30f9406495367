"""Seeded synthetic inputs for the KV-cache epilogue workloads.

This module only draws random numbers and lays out buffers; it holds none of
the epilogue's arithmetic.  The tests (for both the CUDA library and the CPU
oracle) and the benchmark take their inputs from here, so both sides see the
same bytes.

Recipe (numpy ``default_rng``): every tensor draws from its own sub-stream
``default_rng([seed, k])`` with a fixed k per tensor; bf16 and f16 inputs are
round-to-nearest-even conversions of float32 samples (done by torch's cast);
caches are pre-filled with random bytes so that untouched rows are visible;
"fraction p set to -1" means exactly floor(p*T) positions chosen without
replacement; "distinct slots" means ``choice(num_slots, T, replace=False)``.

The shapes and distributions are those of the five workloads the epilogue
is measured on (DeepSeek-V3 MLA shapes for the rmsnorm/rope decode case).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Optional

import numpy as np
import torch

GUARD_BYTES = 256   # random guard band before and after every cache view


def _rng(seed: int, k: int) -> np.random.Generator:
    return np.random.default_rng([seed, k])


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def to_f16_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def to_half_bits(a: np.ndarray, dtype: str) -> np.ndarray:
    return to_bf16_bits(a) if dtype == "bf16" else to_f16_bits(a)


def wide_bf16_bits(rng: np.random.Generator, shape) -> np.ndarray:
    """bf16 bit patterns uniform over all finite values (every exponent, both signs)."""
    bits = rng.integers(0, 1 << 16, size=shape, dtype=np.uint32).astype(np.uint16)
    finite = (bits & 0x7F80) != 0x7F80
    return np.where(finite, bits, bits & 0x807F).astype(np.uint16)


def slots_with_skips(rng: np.random.Generator, num_slots: int, T: int, skip_frac: float,
                     dtype=np.int32) -> np.ndarray:
    s = rng.choice(num_slots, size=T, replace=False).astype(np.int64)
    n_skip = int(np.floor(skip_frac * T))
    if n_skip:
        s[rng.choice(T, size=n_skip, replace=False)] = -1
    return s.astype(dtype)


@dataclass
class CacheBuf:
    """A paged cache [num_blocks, block_size, inner, head_dim] inside a byte buffer.

    The view starts ``offset`` bytes into ``storage``; blocks are
    ``block_stride`` bytes apart (>= block_size*inner*head_dim*elem_bytes when
    the block dimension is strided); random guard bytes surround it.
    """
    storage: np.ndarray
    offset: int
    num_blocks: int
    block_size: int
    inner: int
    head_dim: int
    elem_bytes: int
    block_stride: int

    @property
    def row_bytes(self) -> int:
        return self.inner * self.head_dim * self.elem_bytes

    @property
    def num_slots(self) -> int:
        return self.num_blocks * self.block_size


def make_cache(rng: np.random.Generator, num_blocks: int, block_size: int, head_dim: int,
               elem_bytes: int = 1, inner: int = 1, block_pad_bytes: int = 0,
               guard: int = GUARD_BYTES) -> CacheBuf:
    row = inner * head_dim * elem_bytes
    stride = block_size * row + block_pad_bytes
    nbytes = guard + (num_blocks - 1) * stride + block_size * row + guard
    storage = rng.integers(0, 256, size=nbytes, dtype=np.uint8)
    return CacheBuf(storage, guard, num_blocks, block_size, inner, head_dim, elem_bytes, stride)


# ---------------------------------------------------------------------------
# per-operation generators
# ---------------------------------------------------------------------------
@dataclass
class Case:
    name: str
    op: str
    arrays: Dict[str, np.ndarray] = field(default_factory=dict)
    caches: Dict[str, CacheBuf] = field(default_factory=dict)
    attrs: Dict[str, object] = field(default_factory=dict)


def gen_compress(name: str, T: int, d: int, quant_mode: int, num_blocks: int, block_size: int,
                 head_dim: int, group_size: int = 64, x_scale: float = 1.0, skip_frac: float = 0.0,
                 outlier_frac: float = 0.0, outlier_mult: float = 50.0, seed: int = 0,
                 slot_dtype=np.int32, block_pad_bytes: int = 0, x_kind: str = "normal",
                 guard: int = GUARD_BYTES, x_dtype: str = "bf16") -> Case:
    """x_dtype "f16" (quantMode 0/1): the same samples rounded to float16; the
    "wide" kind then keeps every exponent but the infinity / NaN one."""
    if x_kind == "normal":
        xf = _rng(seed, 1).standard_normal((T, d), dtype=np.float32)
        if outlier_frac > 0:
            rows = _rng(seed, 2).choice(T, size=int(np.floor(outlier_frac * T)), replace=False)
            xf[rows] *= np.float32(outlier_mult)
        x = to_half_bits(xf, x_dtype)
    elif x_kind == "wide":
        x = wide_bf16_bits(_rng(seed, 1), (T, d))
        if x_dtype == "f16":       # the all-ones f16 exponent (inf / NaN) becomes a subnormal
            x = np.where((x & 0x7C00) == 0x7C00, x & 0x83FF, x).astype(np.uint16)
    else:
        raise ValueError(x_kind)
    cache = make_cache(_rng(seed, 3), num_blocks, block_size, head_dim, 1, 1, block_pad_bytes, guard)
    slots = slots_with_skips(_rng(seed, 4), num_blocks * block_size, T, skip_frac, slot_dtype)
    return Case(name, "kv_compress_epilog", {"x": x, "slot_mapping": slots}, {"cache": cache},
                {"quant_mode": quant_mode, "quant_group_size": group_size, "x_scale": x_scale,
                 "x_dtype": x_dtype})


def gen_indexer(name: str, T: int, d: int, quant_mode: int, num_blocks: int, block_size: int,
                cache_head_dim: int, scale_head_dim: int, cache_dtype: str = "e4m3",
                x_dtype: str = "bf16", skip_frac: float = 0.0, seed: int = 0, slot_dtype=np.int32,
                block_pad_bytes: int = 0, x_kind: str = "student_t", guard: int = GUARD_BYTES) -> Case:
    if x_kind == "student_t":
        xf = (0.5 * _rng(seed, 1).standard_t(4, size=(T, d))).astype(np.float32)
        x = to_half_bits(xf, x_dtype)
    elif x_kind == "wide":
        x = wide_bf16_bits(_rng(seed, 1), (T, d))
        if x_dtype == "f16":
            x = (x & 0x8FFF).astype(np.uint16)   # keep f16 finite: exponent field < 31
    else:
        raise ValueError(x_kind)
    scale_elem = 4 if quant_mode == 1 else 1   # fp8 mode keeps a float32 scale per row
    cache = make_cache(_rng(seed, 3), num_blocks, block_size, cache_head_dim, 1, 1, block_pad_bytes, guard)
    cscale = make_cache(_rng(seed, 5), num_blocks, block_size, scale_head_dim, scale_elem, 1,
                        block_pad_bytes, guard)
    slots = slots_with_skips(_rng(seed, 4), num_blocks * block_size, T, skip_frac, slot_dtype)
    return Case(name, "indexer_quant_cache", {"x": x, "slot_mapping": slots},
                {"cache": cache, "cache_scale": cscale},
                {"quant_mode": quant_mode, "cache_dtype": cache_dtype, "x_dtype": x_dtype})


def rope_tables(pos: np.ndarray, dim: int, theta: float = 10000.0):
    """cos/sin [.., dim] from one angle per pair: cat(f(pos*th), f(pos*th)), th_j = theta^(-2j/dim)."""
    j = np.arange(dim // 2, dtype=np.float64)
    inv = theta ** (-2.0 * j / dim)
    ang = pos.astype(np.float64)[..., None] * inv
    c = np.cos(ang)
    s = np.sin(ang)
    return (np.concatenate([c, c], axis=-1).astype(np.float32),
            np.concatenate([s, s], axis=-1).astype(np.float32))


def gen_rmsnorm_rope(name: str, B: int, S: int, D: int, Dv: int, num_blocks: int, block_size: int,
                     k_dtype: str = "bf16", ckv_dtype: str = "e4m3", k_scale=None, ckv_scale=None,
                     k_offset=None, ckv_offset=None, epsilon: float = 1e-6, cache_mode: str = "PA_BNSD",
                     skip_frac: float = 0.0, seed: int = 0, kv_dtype: str = "bf16", slot_dtype=np.int32,
                     block_pad_bytes: int = 0, max_pos: int = 32768, guard: int = GUARD_BYTES) -> Case:
    Dk = D - Dv
    kvf = _rng(seed, 1).standard_normal((B, 1, S, D), dtype=np.float32)
    gamma = (1.0 + 0.1 * _rng(seed, 2).standard_normal(Dv)).astype(np.float32)
    pos = _rng(seed, 6).integers(0, max_pos, size=(B, 1, S))
    cos, sin = rope_tables(pos, Dk)
    eb = {"bf16": 2, "f16": 2, "e4m3": 1, "e5m2": 1, "i8": 1}
    kc = make_cache(_rng(seed, 3), num_blocks, block_size, Dk, eb[k_dtype], 1, block_pad_bytes, guard)
    cc = make_cache(_rng(seed, 5), num_blocks, block_size, Dv, eb[ckv_dtype], 1, block_pad_bytes, guard)
    r = _rng(seed, 4)
    T = B * S
    if cache_mode in ("PA", "PA_BNSD"):
        index = slots_with_skips(r, num_blocks * block_size, T, skip_frac, slot_dtype)
    elif cache_mode == "Norm":
        # index [B, S]: positions inside each batch's cache of block_size rows
        index = np.stack([r.choice(block_size, size=S, replace=False) for _ in range(B)]).astype(np.int64)
        n_skip = int(np.floor(skip_frac * T))
        if n_skip:
            index.reshape(-1)[r.choice(T, size=n_skip, replace=False)] = -1
        index = index.astype(slot_dtype)
    elif cache_mode == "PA_BLK_BNSD":
        nblk = (S + block_size - 1) // block_size
        blocks = r.choice(num_blocks, size=B * nblk, replace=False).astype(np.int64)
        index = blocks * block_size
        n_skip = int(np.floor(skip_frac * index.size))
        if n_skip:
            index[r.choice(index.size, size=n_skip, replace=False)] = -1
        index = index.astype(slot_dtype)
    else:
        raise ValueError(cache_mode)
    arrays = {"kv": to_half_bits(kvf, kv_dtype), "gamma": to_half_bits(gamma, kv_dtype),
              "cos": to_half_bits(cos, kv_dtype).reshape(B, 1, S, Dk),
              "sin": to_half_bits(sin, kv_dtype).reshape(B, 1, S, Dk), "index": index}
    for nm, v in (("k_scale", k_scale), ("ckv_scale", ckv_scale), ("k_offset", k_offset),
                  ("ckv_offset", ckv_offset)):
        if v is not None:
            arrays[nm] = np.asarray(v, dtype=np.float32).reshape(-1)
    return Case(name, "kv_rmsnorm_rope_cache", arrays, {"k_cache": kc, "ckv_cache": cc},
                {"Dv": Dv, "epsilon": epsilon, "cache_mode": cache_mode, "k_dtype": k_dtype,
                 "ckv_dtype": ckv_dtype, "kv_dtype": kv_dtype})


def gen_dequant_rope_quant(name: str, B: int, S: int, Nq: int, Nkv: int, D: int, c0: int, c1: int,
                           x_dtype: str = "i32", x_range: int = 1 << 20, cos_dtype: str = "bf16",
                           cache_mode: str = "page", kv_output: bool = False, with_offsets: bool = True,
                           with_activation_scale: bool = True, bias_dtype: Optional[str] = "f32",
                           skip_frac: float = 0.0, seed: int = 0, x_2d: bool = False,
                           block_pad_bytes: int = 0, guard: int = GUARD_BYTES) -> Case:
    H = (Nq + 2 * Nkv) * D
    if x_dtype == "i32":
        x = _rng(seed, 1).integers(-x_range, x_range, size=(B, S, H), endpoint=True, dtype=np.int64)
        x = x.astype(np.int32)
    else:
        x = to_half_bits(_rng(seed, 1).standard_normal((B, S, H), dtype=np.float32) * 4, x_dtype)
    ws = _rng(seed, 2).uniform(1e-4, 1e-3, size=H).astype(np.float32)
    act = _rng(seed, 7).uniform(0.5, 2.0, size=B * S).astype(np.float32)
    bias_f = (0.1 * _rng(seed, 8).standard_normal(H)).astype(np.float32)
    if bias_dtype == "f32":
        bias = bias_f
    elif bias_dtype in ("bf16", "f16"):
        bias = to_half_bits(bias_f, bias_dtype)
    elif bias_dtype == "i32":
        bias = _rng(seed, 8).integers(-3, 4, size=H).astype(np.int32)
    else:
        bias = None
    pos = np.broadcast_to(np.arange(S)[None, :], (B, S))
    cos, sin = rope_tables(pos, D)
    scale_k = _rng(seed, 9).uniform(0.01, 0.05, size=(Nkv, D)).astype(np.float32)
    scale_v = _rng(seed, 10).uniform(0.01, 0.05, size=(Nkv, D)).astype(np.float32)
    offset_k = _rng(seed, 11).integers(-8, 8, size=(Nkv, D), endpoint=True).astype(np.float32)
    offset_v = _rng(seed, 12).integers(-8, 8, size=(Nkv, D), endpoint=True).astype(np.float32)
    kc = make_cache(_rng(seed, 3), c0, c1, D, 1, Nkv, block_pad_bytes, guard)
    vc = make_cache(_rng(seed, 5), c0, c1, D, 1, Nkv, block_pad_bytes, guard)
    r = _rng(seed, 4)
    if cache_mode == "page":
        idx = slots_with_skips(r, c0 * c1, B * S, skip_frac, np.int32)
    else:
        # one start position per batch: tokens s = 0..S-1 go to start + s
        idx = r.integers(0, c1 - S + 1, size=B).astype(np.int32)
    if x_2d:
        assert S == 1
        x = x.reshape(B, H)
    arrays = {"x": x, "cos": to_half_bits(cos, cos_dtype).reshape(B, S, 1, D),
              "sin": to_half_bits(sin, cos_dtype).reshape(B, S, 1, D), "indices": idx,
              "scale_k": scale_k, "scale_v": scale_v, "weight_scale": ws}
    if with_offsets:
        arrays["offset_k"], arrays["offset_v"] = offset_k, offset_v
    if with_activation_scale:
        arrays["activation_scale"] = act
    if bias is not None:
        arrays["bias"] = bias
    return Case(name, "dequant_rope_quant_kvcache", arrays, {"k_cache": kc, "v_cache": vc},
                {"size_splits": (Nq * D, Nkv * D, Nkv * D), "cache_mode": cache_mode,
                 "kv_output": kv_output, "x_dtype": x_dtype, "cos_dtype": cos_dtype,
                 "bias_dtype": bias_dtype, "Nq": Nq, "Nkv": Nkv, "D": D})


# ---------------------------------------------------------------------------
# the five named workloads (sizes and distributions as specified for them)
# ---------------------------------------------------------------------------
def compress_mode1_T64_d256(seed: int = 0) -> Case:
    return gen_compress("compress_mode1_T64_d256", T=64, d=256, quant_mode=1, num_blocks=8, block_size=16,
                        head_dim=323, skip_frac=0.10, seed=seed)


def rmsnorm_rope_decode_B64_D576(seed: int = 0) -> Case:
    return gen_rmsnorm_rope("rmsnorm_rope_decode_B64_D576", B=64, S=1, D=576, Dv=512, num_blocks=4096, block_size=128,
                            k_dtype="bf16", ckv_dtype="e4m3", ckv_scale=[1.0 / 64.0], epsilon=1e-6,
                            cache_mode="PA_BNSD", skip_frac=0.05, seed=seed)


def indexer_mxfp8_T65536_d128(seed: int = 0) -> Case:
    return gen_indexer("indexer_mxfp8_T65536_d128", T=65536, d=128, quant_mode=0, num_blocks=2048, block_size=64,
                       cache_head_dim=128, scale_head_dim=4, cache_dtype="e4m3", skip_frac=0.05, seed=seed)


def indexer_mxfp4_T65536_d128(seed: int = 0) -> Case:
    return gen_indexer("indexer_mxfp4_T65536_d128", T=65536, d=128, quant_mode=3, num_blocks=2048, block_size=64,
                       cache_head_dim=64, scale_head_dim=4, cache_dtype="u8", skip_frac=0.05, seed=seed)


def dequant_rope_quant_page_B16_S1024_H3072(seed: int = 0, x_range: int = 1 << 20) -> Case:
    return gen_dequant_rope_quant("dequant_rope_quant_page_B16_S1024_H3072", B=16, S=1024, Nq=16, Nkv=4, D=128, c0=512,
                                  c1=128, x_range=x_range, cache_mode="page", seed=seed)


def compress_mode0_T262144_d576(seed: int = 0) -> Case:
    return gen_compress("compress_mode0_T262144_d576", T=262144, d=576, quant_mode=0, num_blocks=4096,
                        block_size=128, head_dim=672, skip_frac=0.02, outlier_frac=0.01, seed=seed)


def compress_mode0_f16_T262144_d576(seed: int = 0) -> Case:
    """The quantMode-0 sweep with float16 x (the page requires bfloat16 only in mode 2)."""
    return gen_compress("compress_mode0_f16_T262144_d576", T=262144, d=576, quant_mode=0, num_blocks=4096,
                        block_size=128, head_dim=672, skip_frac=0.02, outlier_frac=0.01, seed=seed, x_dtype="f16")


def compress_mode2_G32_T262144_d576(seed: int = 0) -> Case:
    return gen_compress("compress_mode2_G32_T262144_d576", T=262144, d=576, quant_mode=2, group_size=32, x_scale=0.1,
                        num_blocks=4096, block_size=128, head_dim=352, skip_frac=0.02, outlier_frac=0.01,
                        seed=seed)


def rmsnorm_rope_prefill_B65536_D576(seed: int = 0) -> Case:
    """The DeepSeek-V3 decode shape (576 = 512 RMSNorm + 64 RoPE columns) at
    prefill size, 65536 tokens, where bandwidth rather than launch latency
    should bound the kernel."""
    return gen_rmsnorm_rope("rmsnorm_rope_prefill_B65536_D576", B=65536, S=1, D=576, Dv=512, num_blocks=1024,
                            block_size=128, k_dtype="bf16", ckv_dtype="e4m3", ckv_scale=[1.0 / 64.0], epsilon=1e-6,
                            cache_mode="PA_BNSD", skip_frac=0.05, seed=seed)


# ---------------------------------------------------------------------------
# the further modes of the four operations at the named workloads' sizes
# ---------------------------------------------------------------------------
def indexer_fp8_T65536_d128(seed: int = 0) -> Case:
    """The mxfp8 indexer rows (65536 x 128) in the fp8 mode: one binary32 scale per row."""
    return gen_indexer("indexer_fp8_T65536_d128", T=65536, d=128, quant_mode=1, num_blocks=2048, block_size=64,
                       cache_head_dim=128, scale_head_dim=1, cache_dtype="e4m3", skip_frac=0.05, seed=seed)


def indexer_mxfp8_e5m2_T65536_d128(seed: int = 0) -> Case:
    """The mxfp8 indexer rows (65536 x 128) into an E5M2 code cache."""
    return gen_indexer("indexer_mxfp8_e5m2_T65536_d128", T=65536, d=128, quant_mode=0, num_blocks=2048, block_size=64,
                       cache_head_dim=128, scale_head_dim=4, cache_dtype="e5m2", skip_frac=0.05, seed=seed)


def rmsnorm_rope_int8_prefill_B65536_D576(seed: int = 0) -> Case:
    """The prefill shape with both caches static int8: per-channel scales
    U(1/48, 1/24) and integer offsets in [-4, 4] for ckv, a per-tensor scale
    1/64 and offset 0 for k."""
    r = _rng(seed, 20)
    return gen_rmsnorm_rope("rmsnorm_rope_int8_prefill_B65536_D576", B=65536, S=1, D=576, Dv=512, num_blocks=1024,
                            block_size=128, k_dtype="i8", ckv_dtype="i8", k_scale=[1.0 / 64.0], k_offset=[0.0],
                            ckv_scale=r.uniform(1.0 / 48.0, 1.0 / 24.0, size=512),
                            ckv_offset=r.integers(-4, 4, size=512, endpoint=True).astype(np.float32),
                            epsilon=1e-6, cache_mode="PA_BNSD", skip_frac=0.05, seed=seed)


def dequant_rope_quant_contiguous_kvout_B16_S1024_H3072(seed: int = 0) -> Case:
    """The page-mode dequant workload (x int32 [16, 1024, 3072]) in contiguous
    cache mode ([16, 2048, 4, 128] caches, each batch's 1024 tokens written
    from its start position) with kOut / vOut."""
    return gen_dequant_rope_quant("dequant_rope_quant_contiguous_kvout_B16_S1024_H3072", B=16, S=1024, Nq=16,
                                  Nkv=4, D=128, c0=16, c1=2048, cache_mode="contiguous", kv_output=True, seed=seed)


def dequant_rope_quant_bf16_page_B16_S1024_H3072(seed: int = 0) -> Case:
    """The page-mode dequant workload's shapes with bf16 x (no dequantisation)."""
    return gen_dequant_rope_quant("dequant_rope_quant_bf16_page_B16_S1024_H3072", B=16, S=1024, Nq=16, Nkv=4,
                                  D=128, c0=512, c1=128, x_dtype="bf16", cos_dtype="bf16", cache_mode="page",
                                  seed=seed)


# ---------------------------------------------------------------------------
# the token Compressor (aclnnCompressor, C128A form: D = 512, coff = 1,
# cmp_ratio = 128; H in the page's 1K..10K range, 7168 as in DeepSeek-V3)
# ---------------------------------------------------------------------------
def gen_compressor(name: str, T: int, H: int, D: int, ratio: int, seed: int = 0, ape_scale: float = 1.0,
                   coff: int = 1) -> Case:
    """x ~ N(0, 1) bf16 [T, H]; W^KV, W^Gate ~ N(0, 1/H) bf16 [coff*D, H] (1/sqrt(H)
    initialisation, so kv_state and score_state are about N(0, 1)); Ape ~
    N(0, ape_scale^2) float32 [ratio, coff*D].  coff 2 (with ratio 4) is the
    C4A / C4Li form."""
    x = to_bf16_bits(_rng(seed, 1).standard_normal((T, H), dtype=np.float32))
    s = np.float32(1.0 / np.sqrt(H))
    wk = to_bf16_bits(_rng(seed, 2).standard_normal((coff * D, H), dtype=np.float32) * s)
    wg = to_bf16_bits(_rng(seed, 3).standard_normal((coff * D, H), dtype=np.float32) * s)
    ape = (_rng(seed, 4).standard_normal((ratio, coff * D), dtype=np.float32) * np.float32(ape_scale)).astype(
        np.float32)
    return Case(name, "compressor", {"x": x, "w_kv": wk, "w_gate": wg, "ape": ape}, {},
                {"ratio": ratio, "coff": coff})


def compressor_c128a_T65536_H7168_D512(seed: int = 0) -> Case:
    return gen_compressor("compressor_c128a_T65536_H7168_D512", T=65536, H=7168, D=512, ratio=128, seed=seed)


def compressor_c128a_T2048_H1024_D512(seed: int = 0) -> Case:
    return gen_compressor("compressor_c128a_T2048_H1024_D512", T=2048, H=1024, D=512, ratio=128, seed=seed)


def compressor_c4a_T65536_H7168_D512(seed: int = 0) -> Case:
    return gen_compressor("compressor_c4a_T65536_H7168_D512", T=65536, H=7168, D=512, ratio=4, seed=seed, coff=2)


def compressor_c4a_T2048_H1024_D512(seed: int = 0) -> Case:
    return gen_compressor("compressor_c4a_T2048_H1024_D512", T=2048, H=1024, D=512, ratio=4, seed=seed, coff=2)


# tensor-core workloads (a dense contraction: timed in TFLOP/s, not HBM bytes)
TENSOR_CONFIGS = {
    "compressor_c128a_T65536_H7168_D512": compressor_c128a_T65536_H7168_D512,
    "compressor_c128a_T2048_H1024_D512": compressor_c128a_T2048_H1024_D512,
    "compressor_c4a_T65536_H7168_D512": compressor_c4a_T65536_H7168_D512,
    "compressor_c4a_T2048_H1024_D512": compressor_c4a_T2048_H1024_D512,
}


CONFIGS = {
    "compress_mode1_T64_d256": compress_mode1_T64_d256,
    "rmsnorm_rope_decode_B64_D576": rmsnorm_rope_decode_B64_D576,
    "rmsnorm_rope_prefill_B65536_D576": rmsnorm_rope_prefill_B65536_D576,
    "indexer_mxfp8_T65536_d128": indexer_mxfp8_T65536_d128,
    "indexer_mxfp4_T65536_d128": indexer_mxfp4_T65536_d128,
    "dequant_rope_quant_page_B16_S1024_H3072": dequant_rope_quant_page_B16_S1024_H3072,
    "compress_mode0_T262144_d576": compress_mode0_T262144_d576,
    "compress_mode2_G32_T262144_d576": compress_mode2_G32_T262144_d576,
    "compress_mode0_f16_T262144_d576": compress_mode0_f16_T262144_d576,
    "indexer_fp8_T65536_d128": indexer_fp8_T65536_d128,
    "indexer_mxfp8_e5m2_T65536_d128": indexer_mxfp8_e5m2_T65536_d128,
    "rmsnorm_rope_int8_prefill_B65536_D576": rmsnorm_rope_int8_prefill_B65536_D576,
    "dequant_rope_quant_contiguous_kvout_B16_S1024_H3072": dequant_rope_quant_contiguous_kvout_B16_S1024_H3072,
    "dequant_rope_quant_bf16_page_B16_S1024_H3072": dequant_rope_quant_bf16_page_B16_S1024_H3072,
}


# ---------------------------------------------------------------------------
# device copies of a case and the library call that updates them
# ---------------------------------------------------------------------------
DEV = "cuda"

TORCH_DT = {"bf16": torch.bfloat16, "f16": torch.float16, "e4m3": torch.float8_e4m3fn,
            "e5m2": torch.float8_e5m2, "i8": torch.int8, "u8": torch.uint8, "e8m0": torch.float8_e8m0fnu,
            "f32": torch.float32}


def half_tensor(bits: np.ndarray, dt: str, device=DEV) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(TORCH_DT[dt]).to(device)


def dev_cache(cb: CacheBuf, dt: torch.dtype):
    st = torch.from_numpy(cb.storage.copy()).to(DEV)
    eb = cb.elem_bytes
    n = (st.numel() - cb.offset) // eb * eb
    typed = st[cb.offset:cb.offset + n].view(dt)
    view = typed.as_strided((cb.num_blocks, cb.block_size, cb.inner, cb.head_dim),
                            (cb.block_stride // eb, cb.inner * cb.head_dim, cb.head_dim, 1))
    return st, view


def f32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def idx(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def shifted(t: torch.Tensor) -> torch.Tensor:
    """The same values in a view that starts one element into a larger buffer
    (so no longer 16-byte aligned), for tests of the unaligned paths."""
    buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
    buf[1:].copy_(t.reshape(-1))
    return buf[1:].view(t.shape)


def build_call(case: Case, misalign: bool = False):
    """Device tensors for a case and a closure that runs the library call once.

    Returns (call, storages, outputs): call(stream=None) enqueues the operation;
    storages maps each cache name to the device copy of its whole byte buffer;
    outputs collects the dense outputs (q_out, k_out, v_out) after a call.
    misalign: dequant_rope_quant_kvcache's x, cos and sin, and
    kv_rmsnorm_rope_cache's cos and sin, start one element past a 16-byte
    boundary.
    """
    import kv_cache_quantize_b200 as kvq
    a, at = case.arrays, case.attrs
    st, views, outs = {}, {}, {}
    if case.op == "kv_compress_epilog":
        st["cache"], views["cache"] = dev_cache(case.caches["cache"], torch.uint8)
        x, s = half_tensor(a["x"], at.get("x_dtype", "bf16")), idx(a["slot_mapping"])

        def call(stream=None):
            kvq.kv_compress_epilog(x, s, views["cache"], at["quant_mode"], at["quant_group_size"], at["x_scale"],
                                   stream=stream)
    elif case.op == "indexer_quant_cache":
        cdt = TORCH_DT[at["cache_dtype"]]
        sdt = torch.float32 if at["quant_mode"] == 1 else torch.float8_e8m0fnu
        st["cache"], views["cache"] = dev_cache(case.caches["cache"], cdt)
        st["cache_scale"], views["cache_scale"] = dev_cache(case.caches["cache_scale"], sdt)
        x, s = half_tensor(a["x"], at["x_dtype"]), idx(a["slot_mapping"])

        def call(stream=None):
            kvq.indexer_quant_cache(x, views["cache"], views["cache_scale"], s, at["quant_mode"], stream=stream)
    elif case.op == "kv_rmsnorm_rope_cache":
        kdt = at["kv_dtype"]
        st["k_cache"], views["k_cache"] = dev_cache(case.caches["k_cache"], TORCH_DT[at["k_dtype"]])
        st["ckv_cache"], views["ckv_cache"] = dev_cache(case.caches["ckv_cache"], TORCH_DT[at["ckv_dtype"]])
        kv = half_tensor(a["kv"], kdt)
        gamma, cos, sin = half_tensor(a["gamma"], kdt), half_tensor(a["cos"], kdt), half_tensor(a["sin"], kdt)
        if misalign:
            cos, sin = shifted(cos), shifted(sin)
        index = idx(a["index"])
        opt = {k: (f32(a[k]) if k in a else None) for k in ("k_scale", "ckv_scale", "k_offset", "ckv_offset")}

        def call(stream=None):
            kvq.kv_rmsnorm_rope_cache(kv, gamma, cos, sin, index, views["k_cache"], views["ckv_cache"],
                                      opt["k_scale"], opt["ckv_scale"], opt["k_offset"], opt["ckv_offset"],
                                      at["epsilon"], at["cache_mode"], stream=stream)
    elif case.op == "dequant_rope_quant_kvcache":
        st["k_cache"], views["k_cache"] = dev_cache(case.caches["k_cache"], torch.int8)
        st["v_cache"], views["v_cache"] = dev_cache(case.caches["v_cache"], torch.int8)
        if at["x_dtype"] == "i32":
            x = torch.from_numpy(np.ascontiguousarray(a["x"])).to(DEV)
        else:
            x = half_tensor(a["x"], at["x_dtype"])
        cos, sin = half_tensor(a["cos"], at["cos_dtype"]), half_tensor(a["sin"], at["cos_dtype"])
        if misalign:
            x, cos, sin = shifted(x), shifted(cos), shifted(sin)
        bias = None
        if "bias" in a:
            bdt = at["bias_dtype"]
            bias = f32(a["bias"]) if bdt == "f32" else (idx(a["bias"]) if bdt == "i32" else half_tensor(a["bias"], bdt))
        opt = {k: (f32(a[k]) if k in a else None)
               for k in ("offset_k", "offset_v", "weight_scale", "activation_scale")}
        sk, sv, ind = f32(a["scale_k"]), f32(a["scale_v"]), idx(a["indices"])

        def call(stream=None):
            q, k, v = kvq.dequant_rope_quant_kvcache(
                x, cos, sin, views["k_cache"], views["v_cache"], ind, sk, sv, opt["offset_k"], opt["offset_v"],
                opt["weight_scale"], opt["activation_scale"], bias, at["size_splits"], "static", "BSND",
                at["kv_output"], at["cache_mode"], outs.get("q_out"), outs.get("k_out"), outs.get("v_out"),
                stream=stream)
            outs["q_out"], outs["k_out"], outs["v_out"] = q, k, v
    elif case.op == "compressor":
        x, wk, wg = half_tensor(a["x"], "bf16"), half_tensor(a["w_kv"], "bf16"), half_tensor(a["w_gate"], "bf16")
        ape = f32(a["ape"])
        outs["cmp_kv"] = torch.empty((a["x"].shape[0] // at["ratio"], a["w_kv"].shape[0] // at.get("coff", 1)),
                                     dtype=torch.bfloat16, device=DEV)

        def call(stream=None):
            kvq.compressor(x, wk, wg, ape, outs["cmp_kv"], at["ratio"], stream=stream)
    else:
        raise ValueError(case.op)
    return call, st, outs
