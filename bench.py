#!/usr/bin/env python
"""Benchmark of the per-token KV-cache epilogue on B200.

A STEP is one pass of the headline workload: kv_compress_epilog over
T = 262144 bf16 token rows of d = 576 (DeepSeek-V3 MLA width), once with
quantMode 0 (group-64 FP8 E4M3 + bf16 scale, 672-byte rows) and once with
quantMode 2 (group-32 FP4 E2M1 + bf16 scale, E4M3 static rope, 352-byte rows),
scattered into paged caches of 4096 blocks x 128 slots (2 % of slots -1, 1 % of
rows x50 outliers).  The two passes read separate copies of x, and every pass
reads 302 MB -- more than the 126 MB L2 -- so no L2 flush is needed.  The
timed region runs the K steps' quantMode-0 passes back to back and then their
quantMode-2 passes, one CUDA event pair around each block (the per-kernel
average launch durations of the roofline come from those events).

value = token rows quantised per second over all ranks (2 x 262144 per step and
GPU); the roofline object reports the dominant kernel's algorithmic HBM bytes
per launch over its CUDA-event duration.  On one GPU every workload is also
timed on its own under "per_config": back-to-back launches cycling through
enough input copies that their bytes exceed twice the L2 size (one copy,
L2-resident, for the latency-bound decode-sized workloads).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--scaling weak|strong]

With N > 1 the script runs under torchrun, one process per GPU; tokens are
independent and each rank owns its caches, so there is no collective on the
data path: by default every rank runs its own copy of the workload (weak
scaling); --scaling strong splits the rows of one workload over the ranks.
The step time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV-epilog tokens/s and achieved HBM GB/s vs ~8 TB/s B200 peak (1 GPU)"
UNIT = "tokens/s"
WORKLOAD = ("kv_compress_epilog large sweep: T=262144 tokens, d=576 bf16 N(0,1) with 1% rows x50; "
            "quantMode=0 (group-64 FP8 E4M3, bf16 scale, 672-B rows) then quantMode=2 (group-32 FP4 E2M1, "
            "bf16 scale, rope FP8 E4M3 static x_scale=0.1, 352-B rows); cache blockSize=128, 4096 blocks; "
            "2% slot_mapping -1")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ---------------------------------------------------------------------------
# algorithmic bytes: what the method must move (each valid row's input bytes
# plus its packed-row bytes out, 4 slot bytes per token, per-token cos/sin and
# activation scale, per-call parameters once); never skipped rows' x, untouched
# cache or headDim tails
# ---------------------------------------------------------------------------
def algorithmic_bytes(case) -> int:
    a, at = case.arrays, case.attrs
    if case.op == "kv_compress_epilog":
        import kv_cache_quantize_b200 as kvq
        T, d = a["x"].shape
        valid = int((a["slot_mapping"] != -1).sum())
        col = kvq.kv_cache_col(d, at["quant_mode"], at["quant_group_size"])
        return valid * (2 * d + col) + T * a["slot_mapping"].itemsize
    if case.op == "indexer_quant_cache":
        import kv_cache_quantize_b200 as kvq
        T, d = a["x"].shape
        valid = int((a["slot_mapping"] != -1).sum())
        mode = at["quant_mode"]
        codes = (d + 1) // 2 if mode == 3 else d
        scales = 4 if mode == 1 else kvq.indexer_scale_col(d, mode)
        return valid * (2 * d + codes + scales) + T * a["slot_mapping"].itemsize
    if case.op == "kv_rmsnorm_rope_cache":
        B, _, S, D = a["kv"].shape
        Dv = at["Dv"]
        Dk = D - Dv
        idx = a["index"]
        valid = int((idx != -1).sum())
        eb = {"bf16": 2, "f16": 2, "e4m3": 1, "e5m2": 1, "i8": 1}
        per_row = 2 * D + 2 * 2 * Dk + Dv * eb[at["ckv_dtype"]] + Dk * eb[at["k_dtype"]]
        params = 2 * Dv + sum(a[k].nbytes for k in ("k_scale", "ckv_scale", "k_offset", "ckv_offset") if k in a)
        return valid * per_row + idx.size * idx.itemsize + params
    if case.op == "dequant_rope_quant_kvcache":
        B, S = a["x"].shape[0], (a["x"].shape[1] if a["x"].ndim == 3 else 1)
        T = B * S
        H = a["x"].shape[-1]
        D, Nq, Nkv = at["D"], at["Nq"], at["Nkv"]
        dq = at["x_dtype"] == "i32"          # the dequant inputs take effect for int32 x only
        per_tok = H * a["x"].itemsize + 2 * 2 * D + Nq * D * 2 + 2 * Nkv * D
        if at["kv_output"]:
            per_tok += 2 * Nkv * D * 2
        per_tok += a["indices"].itemsize if at["cache_mode"] == "page" else 0
        per_tok += 4 if dq and "activation_scale" in a else 0
        used = ("scale_k", "scale_v", "offset_k", "offset_v") + (("weight_scale", "bias") if dq else ())
        params = sum(a[k].nbytes for k in used if k in a)
        if at["cache_mode"] != "page":
            params += a["indices"].nbytes       # one start position per batch
        return T * per_tok + params
    raise ValueError(case.op)


def contraction_flops(case) -> int:
    """FLOPs of the Compressor's two projections (x @ W^KV^T and x @ W^Gate^T):
    2 T H R each for weights of R = coff D rows; the softmax epilogue (a few
    operations per output of the projections) is not counted."""
    T, H = case.arrays["x"].shape
    D = case.arrays["w_kv"].shape[0]
    return 2 * T * H * 2 * D


def bf16_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def token_rows(case) -> int:
    a = case.arrays
    if case.op in ("kv_compress_epilog", "indexer_quant_cache"):
        return int(a["x"].shape[0])
    if case.op == "kv_rmsnorm_rope_cache":
        return int(a["kv"].shape[0] * a["kv"].shape[2])
    return int(a["x"].shape[0] * (a["x"].shape[1] if a["x"].ndim == 3 else 1))


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    """Hash of the CUDA sources with comments and blank lines removed: it
    changes with the code the counters depend on, not with its comments."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kv_cache_quantize_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
        h.update(name.encode() + code.encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str):
    """dram bytes per launch from a committed ncu summary, if taken on the current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    src = kernel_source_hash()
    for line in open(path):
        parts = line.split()
        if len(parts) >= 3 and parts[0] == kernel and parts[1] == src:
            return float(parts[2])
    return None


# ---------------------------------------------------------------------------
# ranks.  Every token row is independent and each rank owns its caches (its
# own sequences' blocks), so ranks exchange nothing on the data path; the
# process group carries only barriers and the max-over-ranks timing.
# ---------------------------------------------------------------------------
def shard_range(n: int, rank: int, world: int):
    """Contiguous share [lo, hi) of n units for rank; shares differ by at most one."""
    q, r = divmod(n, world)
    lo = rank * q + min(rank, r)
    return lo, lo + q + (1 if rank < r else 0)


def rank_workload(make, rank: int, world: int, scaling: str):
    """This rank's part of a compress workload.  weak: a whole copy with the rank's
    own seed (per-GPU work fixed as ranks are added); strong: rows
    shard_range(T, rank, world) of the one seed-0 workload, written into the
    rank's own copy of the cache."""
    if scaling == "weak":
        return make(seed=rank)
    case = make(seed=0)
    T = case.arrays["x"].shape[0]
    lo, hi = shard_range(T, rank, world)
    case.arrays = {"x": case.arrays["x"][lo:hi], "slot_mapping": case.arrays["slot_mapping"][lo:hi]}
    case.name = f"{case.name}[{lo}:{hi}]"
    return case


def max_over_ranks(x: float, dist, device) -> float:
    """The largest x over the ranks of the default process group (x itself alone)."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(n: int, dist, device) -> int:
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return n
    t = torch.tensor([n], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return int(t.item())


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML: the same counters nvidia-smi reads)
# ---------------------------------------------------------------------------
_SAMPLER_CHILD = r"""
import json, select, sys, time
import pynvml
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByUUID(sys.argv[1].encode())
period = float(sys.argv[2])
out = []
first = True
while True:
    t = time.monotonic()
    try:
        out.append((t, pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                    int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))))
    except Exception:
        pass
    if first:                      # NVML is warm: the parent may start its timed work
        sys.stdout.write("ready\n"); sys.stdout.flush()
        first = False
    if select.select([sys.stdin], [], [], period)[0]:
        break
sys.stdout.write(json.dumps(out) + "\n"); sys.stdout.flush()
"""


class ClockSampler:
    """SM clock and throttle reasons of THIS process's GPU, sampled by a child
    process (so the sampling neither competes with the launching thread for the
    interpreter lock nor is starved by it).

    NVML numbers GPUs by physical index and ignores CUDA_VISIBLE_DEVICES, so the
    handle is opened by the CUDA device's UUID (or, failing that, its PCI bus
    id), never by the CUDA ordinal; the UUID is recorded with the samples.
    mark() / mark_end() bracket the timed region on the host's monotonic clock;
    summary() keeps the samples taken inside it."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.0002):
        self.period = period_s
        self.max_mhz = None
        self.uuid = None
        self.samples = []
        self.t0 = self.t1 = None
        self.proc = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            uuid = str(props.uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            except Exception:
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
                u = pynvml.nvmlDeviceGetUUID(h)
                uuid = u.decode() if isinstance(u, bytes) else str(u)
            self.uuid = uuid
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.uuid = None

    def __enter__(self):
        import subprocess
        if self.uuid is not None:
            try:
                self.proc = subprocess.Popen([sys.executable, "-c", _SAMPLER_CHILD, self.uuid, str(self.period)],
                                             stdin=subprocess.PIPE, stdout=subprocess.PIPE, text=True)
                if self.proc.stdout.readline().strip() != "ready":
                    raise RuntimeError("sampler did not start")
            except Exception:
                self.proc = None
        return self

    def mark(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()

    def __exit__(self, *exc):
        if self.proc is not None:
            try:
                out, _ = self.proc.communicate("stop\n", timeout=30)
                self.samples = json.loads(out.strip().splitlines()[-1])
            except Exception:
                self.proc.kill()
                self.samples = []

    def summary(self):
        t0 = self.t0 if self.t0 is not None else float("-inf")
        t1 = self.t1 if self.t1 is not None else float("inf")
        inside = [(m, b) for t, m, b in self.samples if t0 <= t <= t1]
        reasons = sorted({n for _, b in inside for n, bit in self.REASONS.items() if b & bit})
        return {"sm_mhz": statistics.median([m for m, _ in inside]) if inside else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(inside),
                "period_ms": 1e3 * self.period, "gpu_uuid": self.uuid,
                "window_ms": None if self.t0 is None or self.t1 is None else 1e3 * (self.t1 - self.t0)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (the oracle as it stands, all host cores via row chunks)
# ---------------------------------------------------------------------------
def oracle_rows_per_s(cases, budget_s: float, threads: int):
    """Time the oracle on the workload's passes, 16384-row chunk by chunk (alternating
    passes), until budget_s is spent or every row is done; returns (rows/s, rows, s)."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from _oracle_harness import paged
    chunk, rows, spent = 16384, 0, 0.0
    T = min(c.arrays["x"].shape[0] for c in cases)
    for lo in range(0, T, chunk):
        hi = min(T, lo + chunk)
        for case in cases:
            a, at = case.arrays, case.attrs
            st = case.caches["cache"].storage.copy()
            t0 = time.perf_counter()
            oracle.kv_compress_epilog(a["x"][lo:hi], a["slot_mapping"][lo:hi], paged(case.caches["cache"], st),
                                      at["quant_mode"], at["quant_group_size"], at["x_scale"], threads=threads)
            spent += time.perf_counter() - t0
            rows += hi - lo
        if spent >= budget_s:
            break
    return rows / spent, rows, spent


def run_reference(args):
    """The base contract's reference arm: the CPU oracle, timed on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from kv_cache_quantize_b200 import workloads as W
    threads = os.cpu_count() or 1
    cases = [W.compress_mode0_T262144_d576(), W.compress_mode2_G32_T262144_d576()]
    # size each step so that warmup + steps end within about two minutes
    rate, _, _ = oracle_rows_per_s(cases, 2.0, threads)
    per_step_s = min(10.0, 120.0 / max(1, args.steps + args.warmup))
    rows_per_pass = max(256, min(262144, int(rate * per_step_s / 2)))
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from _oracle_harness import paged

    def step():
        for case in cases:
            a, at = case.arrays, case.attrs
            st = case.caches["cache"].storage.copy()
            oracle.kv_compress_epilog(a["x"][:rows_per_pass], a["slot_mapping"][:rows_per_pass],
                                      paged(case.caches["cache"], st), at["quant_mode"], at["quant_group_size"],
                                      at["x_scale"], threads=threads)
    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = 2 * rows_per_pass * args.steps / total
    sample = (f"first {rows_per_pass} of the 262144 token rows of each quantMode pass per step "
              f"(oracle in C, rows split over {threads} host threads)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "parallelism": "cpu oracle, rank 0 only"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def rotation(case, make, l2_bytes: int):
    """Device copies of a workload to cycle through so that consecutive launches
    find their inputs out of L2: enough copies that their algorithmic bytes add
    up to twice the L2 size (at most 16).  Workloads under 4 MB are latency-
    bound and run on one copy (L2-resident)."""
    from kv_cache_quantize_b200 import workloads as W
    nb = algorithmic_bytes(case)
    k = 1 if nb < (4 << 20) else min(16, max(1, -(-2 * l2_bytes // nb)))
    calls = [W.build_call(case)[0]]
    for _ in range(k - 1):
        calls.append(W.build_call(make())[0])
    return calls


def device_us_per_launch(calls, stream, reps: int) -> float:
    """Mean device time of one launch over `reps` back-to-back launches that
    cycle through `calls`.  A device-side wait long enough for the host to
    enqueue every launch precedes the start event, so the events bracket
    device time only (no host call overhead, no idle gaps)."""
    import torch
    t0 = time.perf_counter()
    for i in range(3 * len(calls)):
        calls[i % len(calls)](stream)
    host_s = (time.perf_counter() - t0) / (3 * len(calls))
    torch.cuda.synchronize()
    torch.cuda._sleep(int(2.0e9 * (2.0 * host_s * reps + 50e-6)))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(reps):
        calls[i % len(calls)](stream)
    e1.record(stream)
    torch.cuda.synchronize()
    return 1e3 * e0.elapsed_time(e1) / reps


# the packed-row decoder, timed on the caches of the two headline passes
DECODER_WORKLOADS = {"decompress_mode0_T262144_d576": "compress_mode0_T262144_d576",
                     "decompress_mode2_G32_T262144_d576": "compress_mode2_G32_T262144_d576"}


def decoder_call(case, stream):
    """Encode the case's rows into its cache once, then return (call, algorithmic
    bytes) for decoding them back into a bf16 [T, d] buffer."""
    import numpy as np
    import torch
    import kv_cache_quantize_b200 as kvq
    from kv_cache_quantize_b200 import workloads as W
    call, st, _ = W.build_call(case)
    call(stream)
    cb, at = case.caches["cache"], case.attrs
    view = st["cache"][cb.offset:].as_strided((cb.num_blocks, cb.block_size, 1, cb.head_dim),
                                              (cb.block_stride, cb.head_dim, cb.head_dim, 1))
    slots = torch.from_numpy(np.ascontiguousarray(case.arrays["slot_mapping"])).to(st["cache"].device)
    T, d = case.arrays["x"].shape
    y = torch.empty((T, d), dtype=torch.bfloat16, device=st["cache"].device)

    def dcall(strm):
        kvq.kv_decompress(view, slots, y, at["quant_mode"], at["quant_group_size"], at["x_scale"], stream=strm)
    valid = int((case.arrays["slot_mapping"] != -1).sum())
    col = kvq.kv_cache_col(d, at["quant_mode"], at["quant_group_size"])
    return dcall, valid * (col + 2 * d) + T * case.arrays["slot_mapping"].itemsize


def run_profile_workload(args):
    """Run one named workload a few times (for ncu captures of a single kernel)."""
    import torch
    import kv_cache_quantize_b200 as kvq
    from kv_cache_quantize_b200 import workloads as W
    stream = torch.cuda.current_stream()
    if args.profile_workload in DECODER_WORKLOADS:
        dcall, nb = decoder_call(W.CONFIGS[DECODER_WORKLOADS[args.profile_workload]](), stream)
        us = device_us_per_launch([dcall], stream, args.profile_reps)
        if kvq.get_error(stream) != 0:
            raise RuntimeError("device fault bits set")
        print(f"{args.profile_workload}: {args.profile_reps} launches over 1 input copies, "
              f"{us:.1f} us per launch, {nb / us / 1e3:.0f} GB/s algorithmic")
        return 0
    if args.profile_workload in W.TENSOR_CONFIGS:
        case = W.TENSOR_CONFIGS[args.profile_workload]()
        call, _, _ = W.build_call(case)
        us = device_us_per_launch([call], stream, args.profile_reps)
        if kvq.get_error(stream) != 0:
            raise RuntimeError("device fault bits set")
        print(f"{args.profile_workload}: {args.profile_reps} launches, {us:.1f} us per launch, "
              f"{contraction_flops(case) / us / 1e6:.1f} TFLOP/s")
        return 0
    make = W.CONFIGS[args.profile_workload]
    case = make()
    calls = rotation(case, make, torch.cuda.get_device_properties(0).L2_cache_size)
    us = device_us_per_launch(calls, stream, args.profile_reps)
    if kvq.get_error(stream) != 0:
        raise RuntimeError("device fault bits set")
    print(f"{args.profile_workload}: {args.profile_reps} launches over {len(calls)} input copies, "
          f"{us:.1f} us per launch, {algorithmic_bytes(case) / us / 1e3:.0f} GB/s algorithmic")
    return 0


# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--scaling", default="weak", choices=["weak", "strong"],
                    help="weak: each rank a whole copy of the workload; strong: its rows split over the ranks")
    ap.add_argument("--no-per-config", action="store_true", help="skip the per-workload breakdown")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle timing for cpu_baseline")
    ap.add_argument("--profile-workload", default=None,
                    help="profiling mode: run only this named workload (a workloads.CONFIGS or TENSOR_CONFIGS name, or "
                         "decompress_mode0_T262144_d576 / decompress_mode2_G32_T262144_d576 for the decoder) "
                         "--profile-reps times (back to back, cycling input copies larger than L2) and print its "
                         "time per launch; no JSON line")
    ap.add_argument("--profile-reps", type=int, default=5)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_workload:
        return run_profile_workload(args)

    import numpy as np
    import torch
    import torch.distributed as dist

    import kv_cache_quantize_b200 as kvq
    from kv_cache_quantize_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    kvq.lib()

    # ---------------- headline workload ----------------
    case_a = rank_workload(W.compress_mode0_T262144_d576, rank, world, args.scaling)
    case_b = rank_workload(W.compress_mode2_G32_T262144_d576, rank, world, args.scaling)
    call_a, st_a, _ = W.build_call(case_a)
    call_b, st_b, _ = W.build_call(case_b)
    stream = torch.cuda.current_stream(dev)
    bytes_a, bytes_b = algorithmic_bytes(case_a), algorithmic_bytes(case_b)
    tokens_per_step = token_rows(case_a) + token_rows(case_b)

    # the clock sampler (a child process) starts before the warm-up, so that it
    # is sampling steadily when the timed region begins
    clocks = ClockSampler(local).__enter__()
    for _ in range(args.warmup):
        call_a(stream)
        call_b(stream)
    torch.cuda.synchronize(dev)
    if kvq.get_error(stream) != 0:
        raise RuntimeError("device fault bits set during warm-up")

    # The timed region runs the K quantMode-0 passes back to back, then the K
    # quantMode-2 passes (each pass a whole batch of 262144 rows; the work of K
    # steps).  One event pair brackets each block, so each kernel's average
    # launch duration is measured live while consecutive launches keep their
    # programmatic overlap (an event recorded between two launches would
    # serialise them).
    start, mid, stop = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark()
    start.record(stream)
    for _ in range(args.steps):
        call_a(stream)
    mid.record(stream)
    for _ in range(args.steps):
        call_b(stream)
    stop.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark_end()
    clocks.__exit__(None, None, None)
    elapsed = max_over_ranks(start.elapsed_time(stop) / 1e3, dist, dev)
    tokens_all_ranks = sum_over_ranks(tokens_per_step, dist, dev)
    if world > 1:
        dist.barrier()
    faults = kvq.get_error(stream)

    value = tokens_all_ranks * args.steps / elapsed
    peak, peak_kind = hbm_peak()
    avg_a = start.elapsed_time(mid) / 1e3 / args.steps
    avg_b = mid.elapsed_time(stop) / 1e3 / args.steps
    kernels = {
        "compress_tma_kernel<0,64,2> (quantMode 0)": {
            "alg_bytes_per_launch": bytes_a, "avg_us": 1e6 * avg_a,
            "alg_GBps": bytes_a / avg_a / 1e9, "frac_of_peak": bytes_a / avg_a / 1e9 / peak,
            "share_of_step": avg_a / (avg_a + avg_b)},
        "compress_tma_kernel<2,32,2> (quantMode 2)": {
            "alg_bytes_per_launch": bytes_b, "avg_us": 1e6 * avg_b,
            "alg_GBps": bytes_b / avg_b / 1e9, "frac_of_peak": bytes_b / avg_b / 1e9 / peak,
            "share_of_step": avg_b / (avg_a + avg_b)},
    }
    dom_name, dom_bytes, dom_avg = ("compress_tma_kernel<0,64,2>", bytes_a, avg_a) if avg_a >= avg_b else \
        ("compress_tma_kernel<2,32,2>", bytes_b, avg_b)
    achieved = dom_bytes / dom_avg / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": profiled_traffic(dom_name), "kernel": dom_name,
                "peak_source": f"{peak_kind} hbm_gbs (copy bandwidth)", "alg_bytes_per_launch": dom_bytes}

    # ---------------- end to end through the public API with host buffers ----------------
    e2e_steps = min(args.steps, 10)
    xa_host = torch.from_numpy(case_a.arrays["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    xb_host = torch.from_numpy(case_b.arrays["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    sa_host = torch.from_numpy(case_a.arrays["slot_mapping"]).pin_memory()
    sb_host = torch.from_numpy(case_b.arrays["slot_mapping"]).pin_memory()
    xa_dev, xb_dev = torch.empty_like(xa_host, device=dev), torch.empty_like(xb_host, device=dev)
    sa_dev, sb_dev = torch.empty_like(sa_host, device=dev), torch.empty_like(sb_host, device=dev)
    from kv_cache_quantize_b200.workloads import dev_cache
    _, cache_a = dev_cache(case_a.caches["cache"], torch.uint8)
    _, cache_b = dev_cache(case_b.caches["cache"], torch.uint8)
    at_a, at_b = case_a.attrs, case_b.attrs

    def e2e_step():
        xa_dev.copy_(xa_host, non_blocking=True)
        sa_dev.copy_(sa_host, non_blocking=True)
        kvq.kv_compress_epilog(xa_dev, sa_dev, cache_a, at_a["quant_mode"], at_a["quant_group_size"],
                               at_a["x_scale"], stream=stream)
        xb_dev.copy_(xb_host, non_blocking=True)
        sb_dev.copy_(sb_host, non_blocking=True)
        kvq.kv_compress_epilog(xb_dev, sb_dev, cache_b, at_b["quant_mode"], at_b["quant_group_size"],
                               at_b["x_scale"], stream=stream)
        return kvq.get_error(stream)      # device -> host read of the step's result (fault word)
    for _ in range(3):
        e2e_step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        e2e_step()
    torch.cuda.synchronize(dev)
    e2e_s = time.perf_counter() - t0
    if world > 1:
        t = torch.tensor([e2e_s], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_s = float(t.item())
    h2d = xa_host.nbytes + xb_host.nbytes + sa_host.nbytes + sb_host.nbytes
    e2e = {"value": world * tokens_per_step * e2e_steps / e2e_s, "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": 4, "steps": e2e_steps,
           "note": "pinned host x + slot_mapping copied in, both passes through the C ABI, fault word read back"}
    del xa_host, xb_host, xa_dev, xb_dev, cache_a, cache_b

    # ---------------- per-workload breakdown (single GPU only: with several
    # ranks the others would wait for rank 0 at the final barrier) ----------------
    per_config = None
    per_config_clocks = None
    if rank == 0 and world == 1 and not args.no_per_config:
        per_config = {}
        pc_sampler = ClockSampler(local, 0.005).__enter__()
        pc_sampler.mark()
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        for name, make in W.CONFIGS.items():
            case = {"compress_mode0_T262144_d576": case_a,
                    "compress_mode2_G32_T262144_d576": case_b}.get(name) or make()
            calls = rotation(case, make, l2)
            us = device_us_per_launch(calls, stream, 200)
            nb = algorithmic_bytes(case)
            per_config[name] = {"tokens": token_rows(case), "alg_bytes": nb, "us_per_launch": us,
                                "tokens_per_s": token_rows(case) / us * 1e6, "alg_GBps": nb / us / 1e3,
                                "frac_of_peak": nb / us / 1e3 / peak, "input_copies": len(calls),
                                "l2": ("L2-resident (latency-bound)" if nb < (4 << 20) else
                                       f"{len(calls)} input copies cycled, {len(calls) * nb >> 20} MB > L2")}
            del calls, case
            torch.cuda.empty_cache()
        # the packed-row decoder on the headline caches (written by the timed encoder)
        for name, case in (("decompress_mode0_T262144_d576", case_a), ("decompress_mode2_G32_T262144_d576", case_b)):
            dcall, nb = decoder_call(case, stream)
            us = device_us_per_launch([dcall], stream, 200)
            T = case.arrays["x"].shape[0]
            per_config[name] = {"tokens": T, "alg_bytes": nb, "us_per_launch": us, "tokens_per_s": T / us * 1e6,
                                "alg_GBps": nb / us / 1e3, "frac_of_peak": nb / us / 1e3 / peak,
                                "input_copies": 1, "l2": f"{nb >> 20} MB > L2"}
            del dcall
            torch.cuda.empty_cache()
        # the Compressor (a dense contraction: TFLOP/s against the measured bf16 peak)
        tpeak, tkind = bf16_peak()
        for name, make in W.TENSOR_CONFIGS.items():
            case = make()
            call, _, _ = W.build_call(case)
            us = device_us_per_launch([call], stream, 20)
            fl = contraction_flops(case)
            per_config[name] = {"tokens": int(case.arrays["x"].shape[0]), "flops": fl, "us_per_launch": us,
                                "tokens_per_s": case.arrays["x"].shape[0] / us * 1e6, "TFLOPs": fl / us / 1e6,
                                "frac_of_peak": fl / us / 1e6 / tpeak, "bound": "tensor",
                                "peak_source": f"{tkind} bf16_tflops (burst)",
                                "l2": "x larger than L2" if case.arrays["x"].nbytes > l2 else "L2-resident"}
            del call, case
            torch.cuda.empty_cache()
        # the same access pattern without arithmetic (kvq_scatter_rows): the DRAM
        # ceiling the two compress passes are compared with
        from kv_cache_quantize_b200.workloads import dev_cache
        for name, case in (("scatter_rows_as_mode0_T262144_d576", case_a),
                           ("scatter_rows_as_mode2_G32_T262144_d576", case_b)):
            at = case.attrs
            xt = torch.from_numpy(case.arrays["x"].view(np.int16)).view(torch.bfloat16).to(dev)
            sl = torch.from_numpy(case.arrays["slot_mapping"]).to(dev)
            _, view = dev_cache(case.caches["cache"], torch.uint8)
            col = kvq.kv_cache_col(xt.shape[1], at["quant_mode"], at["quant_group_size"])

            def scall(strm, xt=xt, sl=sl, view=view, col=col):
                kvq.scatter_rows(xt, sl, view, col, stream=strm)
            us = device_us_per_launch([scall], stream, 200)
            nb = algorithmic_bytes(case)
            T = case.arrays["x"].shape[0]
            per_config[name] = {"tokens": T, "alg_bytes": nb, "us_per_launch": us, "tokens_per_s": T / us * 1e6,
                                "alg_GBps": nb / us / 1e3, "frac_of_peak": nb / us / 1e3 / peak,
                                "input_copies": 1, "l2": f"{nb >> 20} MB > L2",
                                "note": "compress access pattern, no arithmetic"}
            del xt, sl, view, scall
            torch.cuda.empty_cache()
        pc_sampler.mark_end()
        pc_sampler.__exit__(None, None, None)
        per_config_clocks = pc_sampler.summary()

    # ---------------- CPU oracle baseline (rank 0, N = 1) ----------------
    cpu = None
    if rank == 0 and world == 1:
        threads = os.cpu_count() or 1
        rate, rows, spent = oracle_rows_per_s([case_a, case_b], args.cpu_budget, threads)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{rows} token rows of the two quantMode passes in 16384-row chunks, {spent:.1f} s "
                         f"(oracle in C, rows split over {threads} host threads)"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": 1e3 * elapsed / args.steps, "higher_is_better": True,
                "scaling": args.scaling, "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": WORKLOAD, "tokens_per_step_per_gpu": tokens_per_step,
                           "alg_bytes_per_step_per_gpu": bytes_a + bytes_b,
                           "alg_GBps_per_gpu": (bytes_a + bytes_b) * args.steps / elapsed / 1e9,
                           "l2": "inputs larger than L2 (two 302 MB x buffers, every pass reads one), no flush",
                           "order": "K quantMode-0 passes back to back, then K quantMode-2 passes; "
                                    "one event pair per block",
                           "parallelism": (f"replicas x{world} (independent token batches, no collective)"
                                           if args.scaling == "weak" else
                                           f"rows split over {world} ranks (own caches, no collective)")},
                "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": 2 * args.steps, "clocks": clocks.summary(), "fault_bits": faults,
                "per_config": per_config, "per_config_clocks": per_config_clocks}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
