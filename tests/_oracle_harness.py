"""Run the CPU oracle on a workloads.Case (test-side glue; no method arithmetic)."""
from __future__ import annotations

import copy

import numpy as np

import oracle
from kv_cache_quantize_b200.workloads import CacheBuf, Case


def paged(c: CacheBuf, storage: np.ndarray) -> oracle.Paged:
    return oracle.Paged(storage, c.offset, c.num_blocks, c.block_size, c.row_bytes, c.block_stride)


def run_oracle(case: Case, threads: int = 1):
    """Returns (dict of updated cache storages, outputs dict, fault bits)."""
    st = {k: v.storage.copy() for k, v in case.caches.items()}
    a, at = case.arrays, case.attrs
    outs = {}
    if case.op == "kv_compress_epilog":
        f = oracle.kv_compress_epilog(a["x"], a["slot_mapping"], paged(case.caches["cache"], st["cache"]),
                                      at["quant_mode"], at["quant_group_size"], at["x_scale"], threads,
                                      x_dtype=at.get("x_dtype", "bf16"))
    elif case.op == "indexer_quant_cache":
        f = oracle.indexer_quant_cache(a["x"], at["x_dtype"], a["slot_mapping"],
                                       paged(case.caches["cache"], st["cache"]),
                                       "e5m2" if at["cache_dtype"] == "e5m2" else "e4m3",
                                       paged(case.caches["cache_scale"], st["cache_scale"]), at["quant_mode"],
                                       threads)
    elif case.op == "kv_rmsnorm_rope_cache":
        kc, cc = case.caches["k_cache"], case.caches["ckv_cache"]
        ko = oracle.CacheOut(paged(kc, st["k_cache"]), at["k_dtype"], a.get("k_scale"), a.get("k_offset"))
        co = oracle.CacheOut(paged(cc, st["ckv_cache"]), at["ckv_dtype"], a.get("ckv_scale"), a.get("ckv_offset"))
        f = oracle.kv_rmsnorm_rope_cache(a["kv"], at["kv_dtype"], at["Dv"], a["gamma"], a["cos"], a["sin"],
                                         a["index"], at["cache_mode"], ko, co, at["epsilon"])
    elif case.op == "dequant_rope_quant_kvcache":
        kc, vc = case.caches["k_cache"], case.caches["v_cache"]
        q, k, v, f = oracle.dequant_rope_quant_kvcache(
            a["x"], at["x_dtype"], a["cos"], a["sin"], at["cos_dtype"], paged(kc, st["k_cache"]),
            paged(vc, st["v_cache"]), a["indices"], a["scale_k"], a["scale_v"], a.get("offset_k"),
            a.get("offset_v"), a.get("weight_scale"), a.get("activation_scale"), a.get("bias"),
            at["bias_dtype"] or "f32", at["size_splits"], at["cache_mode"], at["kv_output"])
        outs = {"q_out": q, "k_out": k, "v_out": v}
    else:
        raise ValueError(case.op)
    return st, outs, f


def row_view(c: CacheBuf, storage: np.ndarray, slot: int, nbytes: int) -> np.ndarray:
    start = c.offset + (slot // c.block_size) * c.block_stride + (slot % c.block_size) * c.row_bytes
    return storage[start:start + nbytes]


def written_mask(c: CacheBuf, slots, nbytes: int) -> np.ndarray:
    """Bytes of the storage that an update of these slots may write (first nbytes of each row)."""
    m = np.zeros(c.storage.size, dtype=bool)
    for s in np.asarray(slots).ravel().tolist():
        if 0 <= s < c.num_slots:
            start = c.offset + (s // c.block_size) * c.block_stride + (s % c.block_size) * c.row_bytes
            m[start:start + nbytes] = True
    return m


def clone_case(case: Case) -> Case:
    return copy.deepcopy(case)
