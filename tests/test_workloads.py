"""The input recipe of the named workloads (CPU only): shapes, dtypes, the
exact number of skipped tokens, distinct destination slots, seeded
reproducibility, and caches pre-filled with random bytes."""
import numpy as np
import pytest

from kv_cache_quantize_b200 import workloads as W

SLOTS = {"kv_compress_epilog": "slot_mapping", "indexer_quant_cache": "slot_mapping",
         "kv_rmsnorm_rope_cache": "index", "dequant_rope_quant_kvcache": "indices"}
SKIP = {"compress_mode1_T64_d256": 0.10, "rmsnorm_rope_decode_B64_D576": 0.05, "indexer_mxfp8_T65536_d128": 0.05,
        "indexer_mxfp4_T65536_d128": 0.05, "dequant_rope_quant_page_B16_S1024_H3072": 0.0,
        "compress_mode0_T262144_d576": 0.02, "compress_mode2_G32_T262144_d576": 0.02,
        "rmsnorm_rope_prefill_B65536_D576": 0.05}


@pytest.mark.parametrize("name", sorted(SKIP))
def test_skips_and_distinct_slots(name):
    case = W.CONFIGS[name]()
    idx = case.arrays[SLOTS[case.op]].reshape(-1)
    n_skip = int(np.floor(SKIP[name] * idx.size))
    assert int((idx == -1).sum()) == n_skip
    live = idx[idx != -1]
    assert np.unique(live).size == live.size                    # every token has its own slot
    assert live.min() >= 0
    first = next(iter(case.caches.values()))
    assert live.max() < first.num_slots


@pytest.mark.parametrize("name", ["compress_mode1_T64_d256", "rmsnorm_rope_decode_B64_D576"])
def test_seeded_and_reproducible(name):
    a, b, c = W.CONFIGS[name](0), W.CONFIGS[name](0), W.CONFIGS[name](1)
    for k in a.arrays:
        assert np.array_equal(a.arrays[k], b.arrays[k]), k
    assert any(not np.array_equal(a.arrays[k], c.arrays[k]) for k in a.arrays)
    for k in a.caches:
        assert np.array_equal(a.caches[k].storage, b.caches[k].storage)


def test_named_shapes():
    c = W.CONFIGS["compress_mode0_T262144_d576"]()
    assert c.arrays["x"].shape == (262144, 576) and c.arrays["x"].dtype == np.uint16
    cb = c.caches["cache"]
    assert (cb.num_blocks, cb.block_size, cb.head_dim) == (4096, 128, 672)
    c = W.CONFIGS["indexer_mxfp8_T65536_d128"]()
    assert c.arrays["x"].shape == (65536, 128)
    c = W.CONFIGS["dequant_rope_quant_page_B16_S1024_H3072"]()
    assert c.arrays["x"].shape == (16, 1024, 3072) and c.arrays["x"].dtype == np.int32
    assert np.abs(c.arrays["x"]).max() <= 1 << 20
    c = W.CONFIGS["rmsnorm_rope_decode_B64_D576"]()
    assert c.arrays["kv"].shape == (64, 1, 1, 576)


def test_caches_start_with_random_bytes():
    """Untouched rows must be visible: the initial cache bytes are not a constant."""
    c = W.CONFIGS["compress_mode1_T64_d256"]()
    st = c.caches["cache"].storage
    assert np.unique(st).size > 200


def test_compressor_inputs():
    """The Compressor's inputs: bf16 x ~ N(0, 1), weights ~ N(0, 1/H), float32 Ape; seeded."""
    c = W.TENSOR_CONFIGS["compressor_c128a_T2048_H1024_D512"]()
    x, wk, wg, ape = (c.arrays[k] for k in ("x", "w_kv", "w_gate", "ape"))
    assert x.shape == (2048, 1024) and x.dtype == np.uint16
    assert wk.shape == wg.shape == (512, 1024) and ape.shape == (128, 512) and ape.dtype == np.float32
    xv = (x.astype(np.uint32) << 16).view(np.float32)
    wv = (wk.astype(np.uint32) << 16).view(np.float32)
    assert abs(float(xv.std()) - 1.0) < 0.01 and abs(float(wv.std()) * 32.0 - 1.0) < 0.02
    assert not np.array_equal(wk, wg)
    d = W.TENSOR_CONFIGS["compressor_c128a_T2048_H1024_D512"]()
    assert all(np.array_equal(c.arrays[k], d.arrays[k]) for k in c.arrays)
