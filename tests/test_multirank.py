"""The multi-rank path of the benchmark on CPU: two gloo ranks (one process
each, rendezvous on 127.0.0.1), the oracle standing in for the GPU kernel.

What is checked: the strong-scaling row shares partition the batch (no row
lost or repeated) and every rank's own cache holds exactly the single-process
result for its rows; the weak-scaling copies are independent seeded batches;
the step time is the maximum over ranks and the token count their sum; the
ranks exchange nothing but these two numbers and barriers.
"""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import oracle  # noqa: E402
from _oracle_harness import paged  # noqa: E402
from kv_cache_quantize_b200 import workloads as W  # noqa: E402


def small(seed=0):
    return W.gen_compress("mr", T=77, d=256, quant_mode=0, num_blocks=12, block_size=16,
                          head_dim=oracle.kv_cache_col(256, 0, 64), skip_frac=0.1, seed=seed)


def _worker(rank, world, port, scaling, out_dir):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    case = bench.rank_workload(small, rank, world, scaling)
    st = case.caches["cache"].storage.copy()
    oracle.kv_compress_epilog(case.arrays["x"], case.arrays["slot_mapping"], paged(case.caches["cache"], st), 0)
    elapsed = bench.max_over_ranks(1.0 + rank, dist, "cpu")
    tokens = bench.sum_over_ranks(int(case.arrays["x"].shape[0]), dist, "cpu")
    np.save(os.path.join(out_dir, f"cache{rank}.npy"), st)
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"elapsed": elapsed, "tokens": tokens, "rows": int(case.arrays["x"].shape[0])}, f)
    dist.barrier()
    dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(scaling, tmp_path, world=2):
    mp.start_processes(_worker, args=(world, _free_port(), scaling, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    caches = [np.load(tmp_path / f"cache{r}.npy") for r in range(world)]
    return res, caches


def test_shard_range_partitions():
    for n in (0, 1, 7, 77, 262144):
        for world in (1, 2, 3, 8):
            spans = [bench.shard_range(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(spans[r][1] == spans[r + 1][0] for r in range(world - 1))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1


def test_strong_scaling_two_ranks(tmp_path):
    res, caches = _run("strong", tmp_path)
    assert [r["elapsed"] for r in res] == [2.0, 2.0]            # max over ranks
    assert [r["tokens"] for r in res] == [77, 77]               # sum over ranks: the whole batch
    assert sum(r["rows"] for r in res) == 77
    full = small(0)
    ref = full.caches["cache"].storage.copy()
    oracle.kv_compress_epilog(full.arrays["x"], full.arrays["slot_mapping"], paged(full.caches["cache"], ref), 0)
    col = oracle.kv_cache_col(256, 0, 64)
    cb = full.caches["cache"]
    for r in range(2):
        lo, hi = bench.shard_range(77, r, 2)
        mine = set(int(s) for s in full.arrays["slot_mapping"][lo:hi] if s >= 0)
        for s in range(cb.num_slots):
            a = cb.offset + (s // cb.block_size) * cb.block_stride + (s % cb.block_size) * cb.row_bytes
            if s in mine:      # the rank's rows: as in the single-process run
                assert np.array_equal(caches[r][a:a + col], ref[a:a + col]), (r, s)
            else:              # everyone else's: untouched in this rank's cache
                assert np.array_equal(caches[r][a:a + col], cb.storage[a:a + col]), (r, s)


def test_weak_scaling_two_ranks(tmp_path):
    res, caches = _run("weak", tmp_path)
    assert [r["elapsed"] for r in res] == [2.0, 2.0]
    assert [r["tokens"] for r in res] == [154, 154]             # two whole copies
    for r in range(2):
        case = small(r)
        ref = case.caches["cache"].storage.copy()
        oracle.kv_compress_epilog(case.arrays["x"], case.arrays["slot_mapping"], paged(case.caches["cache"], ref), 0)
        assert np.array_equal(caches[r], ref)
    assert not np.array_equal(caches[0], caches[1])
