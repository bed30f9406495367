"""Run the CUDA library on a workloads.Case through the C ABI (test-side glue).

Each cache lives in a device copy of the case's whole byte storage (guard bands
and block padding included), so a comparison of the storages checks every byte
the update must and must not write.
"""
from __future__ import annotations

import numpy as np
import torch

import kv_cache_quantize_b200 as kvq
from kv_cache_quantize_b200.workloads import Case, build_call, dev_cache, half_tensor  # noqa: F401


def run_gpu(case: Case, misalign: bool = False):
    """Returns (storages as numpy, 16-bit outputs as uint16 numpy, fault bits)."""
    call, st, outs = build_call(case, misalign)
    kvq.get_error()            # clear stale bits
    call()
    torch.cuda.synchronize()
    faults = kvq.get_error()
    res = {k: v.cpu().numpy() for k, v in st.items()}
    o = {}
    for k, v in outs.items():
        o[k] = None if v is None or v.numel() == 0 else v.view(torch.int16).cpu().numpy().view(np.uint16)
    return res, o, faults
