"""The benchmark's bookkeeping on CPU: the algorithmic byte counts of the named
workloads, and the JSON line of the reference arm (the CPU oracle).

The byte counts follow the rule the roofline uses: each valid row's input bytes
plus its packed-row (or cache-row) bytes out, the index bytes of every row,
per-token cos / sin and activation scales, and each per-call parameter once;
the untouched cache, skipped rows' inputs and headDim tails are never counted.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from kv_cache_quantize_b200 import workloads as W  # noqa: E402

EXPECTED_BYTES = {
    "compress_mode1_T64_d256": 58 * (512 + 323) + 64 * 4,
    # 61 valid tokens x (1152 kv + 256 cos/sin + 512 ckv + 128 k) + 64 x 4 index + 1024 gamma + 4 scale
    "rmsnorm_rope_decode_B64_D576": 61 * 2048 + 64 * 4 + 1024 + 4,
    "indexer_mxfp8_T65536_d128": 62260 * (256 + 128 + 4) + 65536 * 4,
    "indexer_mxfp4_T65536_d128": 62260 * (256 + 64 + 4) + 65536 * 4,
    "dequant_rope_quant_page_B16_S1024_H3072": 16384 * 17928 + 32768,
    "compress_mode0_T262144_d576": 256902 * (1152 + 672) + 262144 * 4,
    "compress_mode2_G32_T262144_d576": 256902 * (1152 + 352) + 262144 * 4,
}


@pytest.mark.parametrize("name", sorted(EXPECTED_BYTES))
def test_algorithmic_bytes_of_the_named_workloads(name):
    assert bench.algorithmic_bytes(W.CONFIGS[name]()) == EXPECTED_BYTES[name]


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                         cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] == 3
    assert line["higher_is_better"] is True and line["vs_baseline"] is None
    assert line["value"] > 0 and line["unit"] == "tokens/s"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert "workload" in line["config"]
