"""Benchmark: FP8 scaled quantization throughput (GB/s of bytes read + written) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the hot path over one batch: a bf16 tensor of 2^30
elements shaped [262144, 4096] (randn with 0.1% of the entries scaled by 1e3,
seed 4 + rank, drawn on the host so that rank 0's tensor is the one the
full-size parity tests compare) quantized to E4M3 with one scale per 1x128
block in a single fused pass (amax, scale, saturating cast, code and scale
stores) and dequantized back to bf16 -- two library launches through the C ABI.
W untimed steps, then exactly K steps between barriers and device syncs, timed
with CUDA events on the launching stream; the max over ranks is reported.
Each kernel moves about 3.25 GB in roughly half a millisecond, so the steps
are launched eagerly with an event after every launch: the events give each
kernel's own duration for the roofline, and their cost (the lost overlap of
one kernel's tail with the next one's start) is inside the timed region.
The inputs (2 GiB in, 1 GiB of codes, 2 GiB out) are far larger than the
126 MB L2, so no flush is needed.

Prints one JSON line (rank 0).  Besides the headline it carries the roofline
of each of the two kernels, the per-mode breakdown (1x128, 128x128, MX,
per-tensor current and delayed with the history update, the transposing
casts, dequant, the size sweep, the consumer GEMM) on the other workload
shapes, the end-to-end figure with host buffers, the CPU oracle as a
baseline, SM clocks sampled during the timed region, and the number of
library launches.

--impl reference times the CPU oracle (the plain C reference) on the same
workload and metric, on a bounded sample of rows per step; rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "quantize GB/s (in+out bytes) and % of B200 HBM roofline per scaling mode"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
LOG2_N = 30
ROWS, COLS = (1 << LOG2_N) // 4096, 4096
BLOCK = (1, 128)
WORKLOAD = ("bf16 tensor of 2^30 elements as [262144, 4096], randn with 0.1% of entries x1e3 (seed 4 + rank); E4M3 "
            "1x128 block quantize in one fused pass (262144x32 fp32 scales) + dequant to bf16")
L2_BYTES = 126 * 1024 * 1024
GRAPH_CHUNK = 1000


def env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def max_over_ranks(values, world: int, device="cuda"):
    """Element-wise max of a list of floats over all ranks (all-reduce MAX); the identity at world == 1."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def step_bytes(rows=ROWS, cols=COLS, br=BLOCK[0], bc=BLOCK[1]):
    """Algorithmic bytes of one step: quantize (read bf16, write codes + scales) + dequant (read codes +
    scales, write bf16)."""
    n = rows * cols
    nscales = math.ceil(rows / br) * math.ceil(cols / bc)
    quant = 2 * n + n + 4 * nscales
    deq = n + 4 * nscales + 2 * n
    return quant, deq


# ---------------------------------------------------------------------------------
# clocks: NVML sampled from a thread while the timed region runs
# ---------------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            # CUDA device numbers may be remapped (CUDA_VISIBLE_DEVICES); NVML is matched by UUID
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = str(e)

    def _sample_once(self):
        self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        try:
            self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            self.reasons |= self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            self._sample_once()
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self._sample_once()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self._thread.join()
            self._sample_once()

    def summary(self):
        if not self.ok:
            return {"error": f"NVML unavailable: {getattr(self, 'err', '?')}"}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "sm_mhz_min": min(self.samples), "reasons": names}


# ---------------------------------------------------------------------------------
# the traffic figure from the committed ncu summary (null once the kernel changed)
# ---------------------------------------------------------------------------------

KERNEL_SOURCES = {
    "k_quant_rowblocks": ["fine_grained_block_b200/csrc/quant_block.cu", "fine_grained_block_b200/csrc/fp8q_device.cuh",
                          "fine_grained_block_b200/csrc/lane_vec.cuh"],
    "k_dequant_flat": ["fine_grained_block_b200/csrc/dequant.cu", "fine_grained_block_b200/csrc/dequant_math.cuh",
                       "fine_grained_block_b200/csrc/fp8q_device.cuh", "fine_grained_block_b200/csrc/lane_vec.cuh"],
}


def source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str):
    """DRAM bytes (read + written) per launch from profiles/traffic_<kernel>.txt, or None once the kernel's
    sources no longer hash to the figure recorded there."""
    path = os.path.join(ROOT, "profiles", f"traffic_{kernel}.txt")
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("source_sha256") != source_hash(kernel):
            return None
        return int(float(kv["dram_bytes_per_launch"]))
    except (OSError, KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------------
# CPU oracle baseline (only bench.py's cpu_baseline leg and --impl reference run it)
# ---------------------------------------------------------------------------------

def oracle_step_seconds(x_rows_bits, reps: int):
    """reps x (1x128 E4M3 quantize + bf16 dequant) of the given rows with the single-threaded C oracle."""
    import oracle
    t0 = time.perf_counter()
    for _ in range(reps):
        q, s = oracle.quantize_blockwise(x_rows_bits, *BLOCK, oracle.E4M3)
        oracle.dequantize(q, oracle.E4M3, s, *BLOCK, out_dtype=oracle.BF16)
    return time.perf_counter() - t0


def oracle_step_seconds_threaded(x_rows_bits, reps: int, threads: int):
    """The same oracle calls, split over 128-row slices (whole blocks) on `threads` threads; the oracle is C
    behind ctypes, which releases the GIL, so the slices run in parallel."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    slices = [x_rows_bits[r:r + 128] for r in range(0, x_rows_bits.shape[0], 128)]

    def one(xs):
        q, s = oracle.quantize_blockwise(xs, *BLOCK, oracle.E4M3)
        oracle.dequantize(q, oracle.E4M3, s, *BLOCK, out_dtype=oracle.BF16)

    with ThreadPoolExecutor(max_workers=threads) as pool:
        t0 = time.perf_counter()
        for _ in range(reps):
            list(pool.map(one, slices))
        return time.perf_counter() - t0


def cpu_baseline_all_cores(bits, budget_s: float = 8.0):
    """The oracle over all host cores (128-row slices in parallel), next to the single-thread figure."""
    threads = max(1, len(os.sched_getaffinity(0)))
    rows = 16384
    xs = bits[:rows]
    t1 = oracle_step_seconds_threaded(xs, 1, threads)
    reps = max(1, int(budget_s / max(t1, 1e-3)))
    t = oracle_step_seconds_threaded(xs, reps, threads)
    qb, db = step_bytes(rows, COLS)
    return {"value": (qb + db) * reps / t / 1e9, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"rows 0-{rows - 1} of the headline tensor (1/16 of it): 1x128 E4M3 quantize + bf16 dequant, "
                      f"the C oracle on {rows // 128} slices of 128 rows over {threads} threads, {reps} reps, "
                      f"{t:.1f} s"}


def cpu_baseline(bits, budget_s: float = 12.0):
    sample_rows = 512
    xs = bits[:sample_rows].copy()
    oracle_step_seconds(xs[:1], 1)  # build + load outside the timing
    t1 = oracle_step_seconds(xs, 1)
    reps = max(1, int(budget_s / max(t1, 1e-3)))
    t = oracle_step_seconds(xs, reps)
    qb, db = step_bytes(sample_rows, COLS)
    return {"value": (qb + db) * reps / t / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"rows 0-{sample_rows - 1} of the headline tensor (1/512 of it): 1x128 E4M3 quantize + bf16 "
                      f"dequant, single-threaded C oracle, {reps} reps, {t:.1f} s"}


def oracle_by_config(args):
    """The CPU oracle's throughput on a sample of each benchmark workload (the handbook's fp32 tensor, the
    4096^2 weight, the 16384x7168 activations, the 8192^2 gradients, the size sweep's 2^30 tensor),
    single-threaded and over every host core (independent row slices in parallel), in GB/s of the same
    algorithmic bytes.  Host only; prints one JSON line."""
    import oracle
    import torch
    from concurrent.futures import ThreadPoolExecutor
    from fine_grained_block_b200 import inputs
    threads = max(1, len(os.sched_getaffinity(0)))
    pool = ThreadPoolExecutor(max_workers=threads)

    def rate(fn, xs, nbytes, budget=args.oracle_budget_s):
        """GB/s of fn over the row slices xs, single-threaded and on all cores."""
        t0 = time.perf_counter()
        fn(xs[0])
        one = time.perf_counter() - t0
        reps = max(1, int(budget / max(one * len(xs), 1e-4)))
        t0 = time.perf_counter()
        for _ in range(reps):
            for x in xs:
                fn(x)
        t1 = time.perf_counter() - t0
        preps = max(1, int(budget / max(t1 / reps / threads, 1e-4)))
        t0 = time.perf_counter()
        for _ in range(preps):
            list(pool.map(fn, xs))
        tn = time.perf_counter() - t0
        return {"one_core": round(nbytes * reps / t1 / 1e9, 4), "all_cores": round(nbytes * preps / tn / 1e9, 3),
                "cores": threads}

    def q_deq(br, bc, fmt, out=oracle.BF16):
        def f(x):
            q, sc = oracle.quantize_blockwise(x, br, bc, fmt)
            oracle.dequantize(q, fmt, sc, br, bc, out_dtype=out)
        return f

    out = {}
    # 1: the handbook's fp32 256x1024 tensor (outliers x1e4), E4M3 per tensor and 1x128, each + dequant
    x1 = inputs.relerr_outlier_tensors()[1][1].numpy()
    n1 = x1.size

    def pt_deq(x):
        q, sc, _ = oracle.quantize_per_tensor(x, oracle.E4M3)
        oracle.dequantize(q, oracle.E4M3, np.array([sc], np.float32), 0, 0, out_dtype=oracle.F32)
    import numpy as np
    out["1_fp32_256x1024_per_tensor_e4m3_and_dequant"] = rate(pt_deq, [x1], 2 * 5 * n1)
    out["1_fp32_256x1024_1x128_e4m3_and_dequant"] = rate(q_deq(1, 128, oracle.E4M3, oracle.F32),
                                                           [x1[r:r + 16] for r in range(0, x1.shape[0], 16)],
                                                           2 * (5 * n1 + 4 * (n1 // 128)))
    # 2: the bf16 4096^2 weight, 128x128 + dequant, on its 32 slices of 128 rows
    w = inputs.bf16_bits(inputs.weight_4096(seed=1))[:4096]
    sl = [w[r:r + 128] for r in range(0, w.shape[0], 128)]
    out["2_bf16_weight_4096_128x128_e4m3_and_dequant"] = rate(q_deq(128, 128, oracle.E4M3), sl,
                                                              2 * (3 * w.size + 4 * (w.size // 16384)))
    # 3: the bf16 activations 16384x7168, 1x128 quantize, on 128-row slices of the first 4096 rows
    a = inputs.bf16_bits(inputs.activation_outlier_channels())[:4096]
    sl = [a[r:r + 128] for r in range(0, a.shape[0], 128)]
    out["3_bf16_activations_16384x7168_1x128_e4m3"] = rate(
        lambda x: oracle.quantize_blockwise(x, 1, 128, oracle.E4M3), sl, 3 * a.size + 4 * (a.size // 128))
    # 4: a delayed E5M2 step of the 8192^2 gradients (cast with the given scale + amax, history update)
    g = inputs.bf16_bits(inputs.gradient_step(inputs.gradient_base(), 20))[:4096]
    sl = [g[r:r + 128] for r in range(0, g.shape[0], 128)]
    h = oracle.AmaxHistory(16, oracle.E5M2)

    def delayed(x):
        _, _, am = oracle.quantize_per_tensor(x, oracle.E5M2, scale=0.5)
        return am
    r4 = rate(delayed, sl, 3 * g.size)
    t0 = time.perf_counter()
    for _ in range(1000):
        h.update(1.0)
    r4["history_update_us"] = round((time.perf_counter() - t0) * 1e3, 3)
    out["4_bf16_gradients_8192x8192_delayed_e5m2"] = r4
    # 5: the headline tensor's first rows: 1x128, 128x128 and per-tensor E5M2, each + dequant
    x5 = inputs.bf16_bits(inputs.sweep_tensor(LOG2_N, seed=4))[:4096]
    sl = [x5[r:r + 128] for r in range(0, x5.shape[0], 128)]
    n5 = x5.size
    out["5_bf16_2^30_1x128_e4m3_and_dequant"] = rate(q_deq(1, 128, oracle.E4M3), sl, 2 * (3 * n5 + 4 * (n5 // 128)))
    out["5_bf16_2^30_128x128_e4m3_and_dequant"] = rate(q_deq(128, 128, oracle.E4M3), sl,
                                                       2 * (3 * n5 + 4 * (n5 // 16384)))

    def pt5(x):
        q, sc, _ = oracle.quantize_per_tensor(x, oracle.E5M2)
        oracle.dequantize(q, oracle.E5M2, np.array([sc], np.float32), 0, 0, out_dtype=oracle.BF16)
    out["5_bf16_2^30_per_tensor_e5m2_and_dequant"] = rate(pt5, sl, 6 * n5)
    print(json.dumps({"oracle_by_config": out, "note": "samples: config 1 whole (per tensor) or in 16-row slices "
                      "(1x128); configs 2-5 the first 4096 rows in 128-row slices; per-tensor slices each take their own amax (the oracle's work per "
                      "element is the same)"}))
    return 0


def run_reference(args):
    rank = env_int("RANK", 0)
    if rank != 0:
        return 0
    import oracle  # noqa: F401  (built on first use)
    from fine_grained_block_b200 import inputs
    bits = inputs.bf16_bits(inputs.sweep_tensor(LOG2_N, seed=4))
    # size each step's sample so that warm-up + K steps take about --ref-budget-s seconds (a minute by default)
    probe = bits[:4].copy()
    oracle_step_seconds(probe, 1)
    t_probe = oracle_step_seconds(probe, 2) / 2
    per_row = t_probe / probe.shape[0]
    budget = args.ref_budget_s / max(1, args.steps + args.warmup)
    rows = int(max(1, min(ROWS, budget / per_row)))
    sample = bits[:rows].copy()
    for _ in range(args.warmup):
        oracle_step_seconds(sample, 1)
    times = [oracle_step_seconds(sample, 1) for _ in range(args.steps)]
    total = sum(times)
    qb, db = step_bytes(rows, COLS)
    value = (qb + db) * args.steps / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "rows": ROWS, "cols": COLS, "block": list(BLOCK), "fmt": "e4m3",
                   "sample_per_step": f"rows 0-{rows - 1} of the seed-4 tensor (whole 1x128 blocks)",
                   "parallelism": "rank 0 only (CPU)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"{rows}x{COLS} rows of the tensor per step, single-threaded C oracle"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------
# the library arm
# ---------------------------------------------------------------------------------

class Raw:
    """Direct C-ABI calls with precomputed arguments (the binding's marshalling, done once)."""

    def __init__(self, stream, lib_path=None):
        from fine_grained_block_b200 import binding
        self.L = binding.load_library(lib_path)
        self.stream = stream.cuda_stream
        self.binding = binding

    def check(self, st, what):
        if st != 0:
            raise RuntimeError(f"{what}: {self.binding.fp8_status_string(st)}")


def time_per_launch(launches, reps, warmup, stream, flush):
    """Mean ms of each launch position over `reps` rounds.

    Every launch is bracketed by CUDA events on `stream`, and an untimed L2 flush (a write of more
    than the L2 size) runs before each launch, so no launch finds its inputs in L2."""
    import torch
    for r in range(warmup):
        for fn in launches:
            fn(r)
    torch.cuda.synchronize()
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in launches]
           for _ in range(reps)]
    for r in range(reps):
        for i, fn in enumerate(launches):
            flush()
            evs[r][i][0].record(stream)
            fn(r)
            evs[r][i][1].record(stream)
    torch.cuda.synchronize()
    return [statistics.fmean(evs[r][i][0].elapsed_time(evs[r][i][1]) for r in range(reps))
            for i in range(len(launches))]


def time_in_graph(launches, reps, dev):
    """Mean ms per round of `launches`, from a CUDA graph of `reps` back-to-back rounds timed with events
    around the whole replay (no events between launches).  Used for tensors larger than L2, where each
    launch finds its inputs in HBM without a flush."""
    import torch
    cap = torch.cuda.Stream(dev)
    for r in range(2):
        for fn in launches:
            fn(r, torch.cuda.current_stream(dev).cuda_stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        cs = torch.cuda.current_stream().cuda_stream
        for r in range(reps):
            for fn in launches:
                fn(r, cs)
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) / reps


def modes_breakdown(dev, stream, peak):
    """GB/s of each scaling mode on its own workload shape (one GPU, outside the headline timing)."""
    import torch
    from fine_grained_block_b200 import inputs
    raw = Raw(stream)
    L = raw.L
    out = {}

    def put(name, workload, nbytes, ms):
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"workload": workload, "GB_s": round(gbs, 1), "frac_of_peak": round(gbs / peak, 4),
                     "us": round(ms * 1e3, 2)}

    # 1x128 E4M3, activations 16384x7168 with 8 outlier channels (224 MiB in, > L2)
    a = inputs.activation_outlier_channels(device=dev)
    R_, C_ = a.shape
    n = a.numel()
    q = torch.empty(a.shape, dtype=torch.uint8, device=dev)
    s = torch.empty(R_, C_ // 128, dtype=torch.float32, device=dev)
    y = torch.empty(a.shape, dtype=torch.bfloat16, device=dev)
    wl = "bf16 activations 16384x7168, 8 channels x1e3, seed 2"
    put("1x128_e4m3_quant", wl, 3 * n + 4 * (n // 128), time_in_graph([lambda r, st: raw.check(
        L.fp8_quantize_blockwise(a.data_ptr(), 1, R_, C_, 1, 128, 0, q.data_ptr(), s.data_ptr(), st), "1x128")],
        20, dev))
    put("1x128_dequant_bf16", wl, 3 * n + 4 * (n // 128), time_in_graph([lambda r, st: raw.check(
        L.fp8_dequantize(q.data_ptr(), 0, R_, C_, 1, 128, s.data_ptr(), y.data_ptr(), 1, st), "dequant")], 20, dev))
    put("1x128_fake_quant_bf16", wl + " (one pass, bf16 -> bf16, no codes written)", 4 * n, time_in_graph([
        lambda r, st: raw.check(L.fp8_fake_quantize(a.data_ptr(), 1, R_, C_, 1, 128, 0, None, y.data_ptr(), None,
                                                    st), "fake quant")], 20, dev))
    # MX (1x32 blocks, E8M0 byte scales, fit rule) on the same activations
    e8 = torch.empty(R_, C_ // 32, dtype=torch.uint8, device=dev)
    put("mx1x32_e4m3_quant", wl, 3 * n + n // 32, time_in_graph([lambda r, st: raw.check(
        L.fp8_quantize_mx(a.data_ptr(), 1, R_, C_, 0, 0, q.data_ptr(), e8.data_ptr(), st), "mx")], 20, dev))
    put("mx1x32_dequant_bf16", wl, 3 * n + n // 32, time_in_graph([lambda r, st: raw.check(
        L.fp8_dequantize_mx(q.data_ptr(), 0, R_, C_, e8.data_ptr(), y.data_ptr(), 1, st), "mx dequant")], 20, dev))
    # per-tensor with a transposed copy (q and qt), delayed scale (one pass: 2 B read + 2 B written per element)
    # and current scaling (amax pass first)
    qt = torch.empty(C_, R_, dtype=torch.uint8, device=dev)
    sc = torch.full((1,), 0.25, dtype=torch.float32, device=dev)
    so_ = torch.empty(1, dtype=torch.float32, device=dev)
    ao_ = torch.empty(1, dtype=torch.float32, device=dev)
    put("per_tensor_transpose_delayed_e4m3", wl + " (q and qt, one pass with amax)", 4 * n, time_in_graph([
        lambda r, st: raw.check(L.fp8_quantize_per_tensor_transpose(a.data_ptr(), 1, R_, C_, 0, sc.data_ptr(),
                                                                    q.data_ptr(), qt.data_ptr(), so_.data_ptr(),
                                                                    ao_.data_ptr(), st), "transpose")], 20, dev))
    a2 = a.clone()  # alternate two copies: the reverse cast pass ends where the next amax pass starts
    aa = [a, a2]
    put("per_tensor_transpose_current_e4m3", wl + " (amax pass, then q and qt; alg bytes 4/elem; two input "
        "copies alternated)", 4 * n, time_in_graph([lambda r, st: raw.check(L.fp8_quantize_per_tensor_transpose(
            aa[r % 2].data_ptr(), 1, R_, C_, 0, None, q.data_ptr(), qt.data_ptr(), so_.data_ptr(), ao_.data_ptr(),
            st), "transpose")], 20, dev))
    del a2, aa
    # 1x128 blocks of x and of x^T (the operand of the weight-gradient GEMM) from one read: q with row-block
    # scales, qt with column-block scales
    sbt = torch.empty(C_, R_ // 128, dtype=torch.float32, device=dev)
    put("1x128_e4m3_quant_and_transpose", wl + " (q with 1x128 row-block scales and qt = 1x128 blocks of x^T, "
        "one pass)", 4 * n + 8 * (n // 128), time_in_graph([lambda r, st: raw.check(
            L.fp8_quantize_blockwise_transpose(a.data_ptr(), 1, R_, C_, 1, 128, 0, q.data_ptr(), s.data_ptr(),
                                               qt.data_ptr(), sbt.data_ptr(), st), "block transpose")], 20, dev))
    s2_ = torch.empty(R_ // 128, C_ // 128, dtype=torch.float32, device=dev)
    st2_ = torch.empty(C_ // 128, R_ // 128, dtype=torch.float32, device=dev)
    put("128x128_e4m3_quant_and_transpose", wl + " (q and qt = q^T with 128x128 tile scales, one pass)",
        4 * n + 8 * (n // 16384), time_in_graph([lambda r, st: raw.check(
            L.fp8_quantize_blockwise_transpose(a.data_ptr(), 1, R_, C_, 128, 128, 0, q.data_ptr(), s2_.data_ptr(),
                                               qt.data_ptr(), st2_.data_ptr(), st), "block transpose")], 20, dev))
    del sbt, s2_, st2_
    del a, q, s, y, e8, qt

    # size sweep point 2^28 (512 MiB bf16): 1x128, 128x128, per-tensor current E5M2, dequant
    x = inputs.sweep_tensor(28, device=dev)
    R, C = x.shape
    n = x.numel()
    q = torch.empty(R, C, dtype=torch.uint8, device=dev)
    s1 = torch.empty(R, C // 128, dtype=torch.float32, device=dev)
    s2 = torch.empty(R // 128, C // 128, dtype=torch.float32, device=dev)
    so = torch.empty(1, dtype=torch.float32, device=dev)
    ao = torch.empty(1, dtype=torch.float32, device=dev)
    y = torch.empty(R, C, dtype=torch.bfloat16, device=dev)
    wl = "bf16 randn 2^28 as [65536, 4096], 0.1% x1e3, seed 4"
    put("sweep2^28_1x128_e4m3_quant", wl, 3 * n + 4 * (n // 128), time_in_graph([lambda r, st: raw.check(
        L.fp8_quantize_blockwise(x.data_ptr(), 1, R, C, 1, 128, 0, q.data_ptr(), s1.data_ptr(), st), "1x128")],
        10, dev))
    put("sweep2^28_128x128_e4m3_quant", wl, 3 * n + 4 * (n // 16384), time_in_graph([lambda r, st: raw.check(
        L.fp8_quantize_blockwise(x.data_ptr(), 1, R, C, 128, 128, 0, q.data_ptr(), s2.data_ptr(), st), "128x128")],
        10, dev))
    x2 = x.clone()  # alternate two copies: the cast pass ends where the next amax pass starts
    xa = [x, x2]
    put("sweep2^28_per_tensor_current_e5m2", wl + " (two passes: amax, then cast; alg bytes 3/elem)", 3 * n,
        time_in_graph([lambda r, st: raw.check(L.fp8_quantize_per_tensor(
            xa[r % 2].data_ptr(), 1, n, 1, None, q.data_ptr(), so.data_ptr(), ao.data_ptr(), st), "per-tensor")],
            10, dev))
    del x2, xa
    put("sweep2^28_per_tensor_dequant_bf16", wl, 3 * n, time_in_graph([lambda r, st: raw.check(
        L.fp8_dequantize(q.data_ptr(), 1, R, C, 0, 0, so.data_ptr(), y.data_ptr(), 1, st), "dequant")], 10, dev))
    del x, q, s1, s2, y

    # delayed scaling E5M2, gradient 8192x8192, window 16: cast + amax in one pass, then the history update
    base = inputs.gradient_base(device=dev)
    gs = [inputs.gradient_step(base, k) for k in range(2)]  # 2 x 128 MiB, alternated
    del base
    n = gs[0].numel()
    q = torch.empty(gs[0].shape, dtype=torch.uint8, device=dev)
    hist = torch.zeros(16, dtype=torch.float32, device=dev)
    state = torch.zeros(2, dtype=torch.int32, device=dev)
    scale = torch.ones(1, dtype=torch.float32, device=dev)
    used = torch.empty(1, dtype=torch.float32, device=dev)
    amax = torch.empty(1, dtype=torch.float32, device=dev)
    fq = lambda r, st: raw.check(L.fp8_quantize_per_tensor(gs[r % 2].data_ptr(), 1, n, 1, scale.data_ptr(),
                                                           q.data_ptr(), used.data_ptr(), amax.data_ptr(), st),
                                 "delayed")
    fh = lambda r, st: raw.check(L.fp8_amax_history_update(hist.data_ptr(), state.data_ptr(), 16, amax.data_ptr(), 1,
                                                           scale.data_ptr(), st), "history")
    t_step = time_in_graph([fq, fh], 32, dev)
    t_hist = time_in_graph([fh], 64, dev)
    put("delayed_e5m2_step", "bf16 gradients 8192x8192, |g| log-uniform [1e-6,1e-2], seed 3, W=16 "
        "(cast + amax in one pass, then the history update)", 3 * n, t_step)
    out["delayed_e5m2_history_update_us"] = round(t_hist * 1e3, 2)
    ws = torch.zeros(4, dtype=torch.int32, device=dev)
    fs = lambda r, st: raw.check(L.fp8_quantize_delayed_step(
        gs[r % 2].data_ptr(), 1, n, 1, scale.data_ptr(), hist.data_ptr(), state.data_ptr(), 16, 0, 1.0, 1.0,
        q.data_ptr(), used.data_ptr(), amax.data_ptr(), ws.data_ptr(), st), "delayed step")
    put("delayed_e5m2_step_one_launch", "bf16 gradients 8192x8192, |g| log-uniform [1e-6,1e-2], seed 3, W=16 "
        "(cast + amax + history update in one launch: the last CTA updates)", 3 * n, time_in_graph([fs], 32, dev))
    del gs, q

    # the consumer: blockwise-scaled FP8 GEMM on the tensor cores, 1x128 activations x 128x128 weights
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
        bf16_peak, peak_kind = float(peaks["bf16_tflops"]), "measured bf16 burst x 2 (nominal fp8/bf16)"
        bf16_sustained = float(peaks.get("bf16_tflops_sustained", bf16_peak))
    except (OSError, KeyError, ValueError):
        bf16_peak, peak_kind = 1590.0, "fallback bf16 x 2 (nominal fp8/bf16)"
        bf16_sustained = 1400.0  # the fallback's figure for a GEMM held under the power cap
    fp8_peak = 2.0 * bf16_peak
    fp8_sustained = 2.0 * bf16_sustained
    st0 = stream.cuda_stream
    for (Mg, Ng, Kg) in ((4096, 4096, 4096), (16384, 4096, 7168)):
        xg = inputs.random_matrix(Mg, Kg, seed=6, dtype=torch.bfloat16, outlier_frac=1e-3, factor=1e2, device=dev)
        wg = inputs.random_matrix(Ng, Kg, seed=7, dtype=torch.bfloat16, scale=0.02, device=dev)
        qa = torch.empty(Mg, Kg, dtype=torch.uint8, device=dev)
        sa = torch.empty(Mg, Kg // 128, dtype=torch.float32, device=dev)
        qb = torch.empty(Ng, Kg, dtype=torch.uint8, device=dev)
        sb = torch.empty(Ng // 128, Kg // 128, dtype=torch.float32, device=dev)
        raw.check(L.fp8_quantize_blockwise(xg.data_ptr(), 1, Mg, Kg, 1, 128, 0, qa.data_ptr(), sa.data_ptr(), st0),
                  "1x128")
        raw.check(L.fp8_quantize_blockwise(wg.data_ptr(), 1, Ng, Kg, 128, 128, 0, qb.data_ptr(), sb.data_ptr(), st0),
                  "128x128")
        cg = torch.empty(Mg, Ng, dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize()
        del xg, wg
        ms = time_in_graph([lambda r, st: raw.check(L.fp8_gemm_blockwise(
            qa.data_ptr(), sa.data_ptr(), 0, qb.data_ptr(), sb.data_ptr(), 0, Mg, Ng, Kg, cg.data_ptr(), 1, st),
            "gemm")], 10, dev)
        tflops = 2.0 * Mg * Ng * Kg / (ms * 1e-3) / 1e12
        out[f"gemm_blockwise_e4m3_{Mg}x{Ng}x{Kg}"] = {
            "workload": f"A [{Mg}, {Kg}] 1x128-scaled E4M3 x B [{Ng}, {Kg}] 128x128-scaled E4M3 -> bf16",
            "TFLOP_s": round(tflops, 1), "frac_of_peak": round(tflops / fp8_peak, 4), "peak_TFLOP_s": fp8_peak,
            "peak_kind": peak_kind, "frac_of_sustained_peak": round(tflops / fp8_sustained, 4),
            "sustained_peak_TFLOP_s": fp8_sustained, "us": round(ms * 1e3, 2)}
        del qa, sa, qb, sb, cg

    # the weight-gradient GEMM of the same layer: dW [4096, 7168] = dY^T [4096, 16384] X [16384, 7168], both
    # operands 1x128 along the 16384 tokens (the transposed outputs of fp8_quantize_blockwise_transpose)
    Mg, Ng, Kg = 4096, 7168, 16384
    dyt = inputs.random_matrix(Mg, Kg, seed=8, dtype=torch.bfloat16, scale=1e-3, outlier_frac=1e-3, factor=1e2,
                               device=dev)
    xt = inputs.random_matrix(Ng, Kg, seed=9, dtype=torch.bfloat16, outlier_frac=1e-3, factor=1e2, device=dev)
    qa = torch.empty(Mg, Kg, dtype=torch.uint8, device=dev)
    sa = torch.empty(Mg, Kg // 128, dtype=torch.float32, device=dev)
    qb = torch.empty(Ng, Kg, dtype=torch.uint8, device=dev)
    sb = torch.empty(Ng, Kg // 128, dtype=torch.float32, device=dev)
    raw.check(L.fp8_quantize_blockwise(dyt.data_ptr(), 1, Mg, Kg, 1, 128, 1, qa.data_ptr(), sa.data_ptr(), st0),
              "1x128")
    raw.check(L.fp8_quantize_blockwise(xt.data_ptr(), 1, Ng, Kg, 1, 128, 0, qb.data_ptr(), sb.data_ptr(), st0),
              "1x128")
    cg = torch.empty(Mg, Ng, dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    del dyt, xt
    ms = time_in_graph([lambda r, st: raw.check(L.fp8_gemm_blockwise_ex(
        qa.data_ptr(), sa.data_ptr(), 1, qb.data_ptr(), sb.data_ptr(), 1, 0, Mg, Ng, Kg, cg.data_ptr(), 1, st),
        "gemm wgrad")], 10, dev)
    tflops = 2.0 * Mg * Ng * Kg / (ms * 1e-3) / 1e12
    out[f"gemm_weight_gradient_e5m2xe4m3_{Mg}x{Ng}x{Kg}"] = {
        "workload": f"dY^T [{Mg}, {Kg}] 1x128-scaled E5M2 x X^T [{Ng}, {Kg}] 1x128-scaled E4M3 -> bf16 dW",
        "TFLOP_s": round(tflops, 1), "frac_of_peak": round(tflops / fp8_peak, 4), "peak_TFLOP_s": fp8_peak,
        "peak_kind": peak_kind, "frac_of_sustained_peak": round(tflops / fp8_sustained, 4),
        "sustained_peak_TFLOP_s": fp8_sustained, "us": round(ms * 1e3, 2)}
    del qa, sa, qb, sb, cg

    # many small tensors: 128 weights of 1024x1024 bf16 (2^20 elements each, 256 MiB in all), 128x128 E4M3,
    # one call per tensor against one grouped call
    from fine_grained_block_b200.binding import FP8BlockTensor
    ws_ = [inputs.random_matrix(1024, 1024, seed=100 + i, dtype=torch.bfloat16, scale=0.02, device=dev)
           for i in range(128)]
    wq_ = [torch.empty(1024, 1024, dtype=torch.uint8, device=dev) for _ in ws_]
    wsc_ = [torch.empty(8, 8, dtype=torch.float32, device=dev) for _ in ws_]
    arr = (FP8BlockTensor * len(ws_))(*[FP8BlockTensor(w.data_ptr(), q_.data_ptr(), s_.data_ptr(), 1024, 1024)
                                        for w, q_, s_ in zip(ws_, wq_, wsc_)])
    nb = sum(3 * w.numel() + 4 * 64 for w in ws_)

    def one_by_one(r, st):
        for w, q_, s_ in zip(ws_, wq_, wsc_):
            raw.check(L.fp8_quantize_blockwise(w.data_ptr(), 1, 1024, 1024, 128, 128, 0, q_.data_ptr(), s_.data_ptr(),
                                               st), "128x128")
    put("128_weights_1024x1024_128x128_one_call_each", "128 bf16 weights 1024x1024, N(0,0.02^2), seeds 100..227 "
        "(128 launches)", nb, time_in_graph([one_by_one], 4, dev))
    put("128_weights_1024x1024_128x128_grouped", "the same 128 weights in one fp8_quantize_blockwise_grouped call "
        "(1 launch)", nb, time_in_graph([lambda r, st: raw.check(L.fp8_quantize_blockwise_grouped(
            arr, len(ws_), 1, 128, 128, 0, st), "grouped")], 16, dev))
    del ws_, wq_, wsc_, arr

    # many small per-tensor delayed steps: 128 bf16 gradients of 2^20 elements, E5M2, W=16; one
    # fp8_quantize_delayed_step per tensor against one grouped call
    from fine_grained_block_b200.binding import FP8DelayedTensor
    gx_ = [inputs.random_matrix(1, 1 << 20, seed=300 + i, dtype=torch.bfloat16, scale=1e-3, device=dev).reshape(-1)
           for i in range(128)]
    gq_ = [torch.empty(1 << 20, dtype=torch.uint8, device=dev) for _ in gx_]
    gst_ = [(torch.ones(1, device=dev), torch.zeros(16, device=dev), torch.zeros(2, dtype=torch.int32, device=dev),
             torch.empty(1, device=dev), torch.empty(1, device=dev)) for _ in gx_]
    gws_ = torch.zeros(len(gx_) * 4, dtype=torch.int32, device=dev)
    garr = (FP8DelayedTensor * len(gx_))(*[FP8DelayedTensor(x_.data_ptr(), q_.data_ptr(), x_.numel(), sc_.data_ptr(),
                                                            h_.data_ptr(), stt_.data_ptr(), su_.data_ptr(),
                                                            am_.data_ptr())
                                           for x_, q_, (sc_, h_, stt_, su_, am_) in zip(gx_, gq_, gst_)])
    gnb = 3 * sum(x_.numel() for x_ in gx_)

    def steps_one_by_one(r, st):
        for i, (x_, q_, (sc_, h_, stt_, su_, am_)) in enumerate(zip(gx_, gq_, gst_)):
            raw.check(L.fp8_quantize_delayed_step(x_.data_ptr(), 1, x_.numel(), 1, sc_.data_ptr(), h_.data_ptr(),
                                                  stt_.data_ptr(), 16, 0, 1.0, 1.0, q_.data_ptr(), su_.data_ptr(),
                                                  am_.data_ptr(), gws_[4 * i:4 * i + 4].data_ptr(), st), "step")
    put("128_gradients_2^20_delayed_e5m2_one_call_each", "128 bf16 tensors of 2^20 elements, N(0,1e-6), seeds "
        "300..427, W=16 (128 launches)", gnb, time_in_graph([steps_one_by_one], 4, dev))
    put("128_gradients_2^20_delayed_e5m2_grouped", "the same 128 tensors in one fp8_quantize_delayed_step_grouped "
        "call (1 launch)", gnb, time_in_graph([lambda r, st: raw.check(
            L.fp8_quantize_delayed_step_grouped(garr, len(gx_), 1, 1, 16, 0, 1.0, 1.0, gws_.data_ptr(), st),
            "grouped step")], 16, dev))
    del gx_, gq_, gst_, gws_, garr

    # many small per-tensor current-scaling casts: 128 bf16 tensors of 2^20 elements, E4M3, each with its own
    # amax and scale; one fp8_quantize_per_tensor call per tensor against one grouped call (3 launches)
    from fine_grained_block_b200.binding import FP8CurrentTensor
    cx_ = [inputs.random_matrix(1, 1 << 20, seed=500 + i, dtype=torch.bfloat16, outlier_frac=1e-3, factor=1e3,
                                device=dev).reshape(-1) for i in range(128)]
    cq_ = [torch.empty(1 << 20, dtype=torch.uint8, device=dev) for _ in cx_]
    cs_ = torch.empty(len(cx_), dtype=torch.float32, device=dev)
    ca_ = torch.empty(len(cx_), dtype=torch.float32, device=dev)
    carr = (FP8CurrentTensor * len(cx_))(*[FP8CurrentTensor(x_.data_ptr(), q_.data_ptr(), x_.numel(),
                                                            cs_[i:i + 1].data_ptr(), ca_[i:i + 1].data_ptr())
                                           for i, (x_, q_) in enumerate(zip(cx_, cq_))])
    cnb = 3 * sum(x_.numel() for x_ in cx_)

    def current_one_by_one(r, st):
        for i, (x_, q_) in enumerate(zip(cx_, cq_)):
            raw.check(L.fp8_quantize_per_tensor(x_.data_ptr(), 1, x_.numel(), 0, None, q_.data_ptr(),
                                                cs_[i:i + 1].data_ptr(), ca_[i:i + 1].data_ptr(), st), "per-tensor")
    put("128_tensors_2^20_per_tensor_current_e4m3_one_call_each", "128 bf16 tensors of 2^20 elements, N(0,1) with "
        "0.1% x1e3, seeds 500..627 (128 x 3 launches; alg bytes 3/elem)", cnb, time_in_graph([current_one_by_one], 4,
                                                                                           dev))
    put("128_tensors_2^20_per_tensor_current_e4m3_grouped", "the same 128 tensors in one "
        "fp8_quantize_per_tensor_grouped call (3 launches; alg bytes 3/elem)", cnb, time_in_graph([
            lambda r, st: raw.check(L.fp8_quantize_per_tensor_grouped(carr, len(cx_), 1, 0, st), "grouped current")],
            16, dev))
    del cx_, cq_, cs_, ca_, carr

    # size sweep 2^20 .. 2^30 elements (bf16, 0.1% x1e3 outliers, seed 4): GB/s per mode and size.  Sizes
    # whose buffers fit in L2 rotate over enough copies that every launch reads from HBM.
    sweep = {}
    for lg in (20, 22, 24, 26, 28, 30):
        x0 = inputs.sweep_tensor(lg, device=dev)
        R, C = x0.shape
        n = x0.numel()
        set_bytes = 2 * n + n + 4 * (n // 128) + 2 * n
        copies = max(1, math.ceil(3 * L2_BYTES / set_bytes))
        xs_ = [x0] + [x0.clone() for _ in range(copies - 1)]
        qs_ = [torch.empty(R, C, dtype=torch.uint8, device=dev) for _ in range(copies)]
        ss_ = [torch.empty(R, C // 128, dtype=torch.float32, device=dev) for _ in range(copies)]
        st_ = [torch.empty(R // 128 if R >= 128 else 1, C // 128, dtype=torch.float32, device=dev)
               for _ in range(copies)]
        ys_ = [torch.empty(R, C, dtype=torch.bfloat16, device=dev) for _ in range(copies)]
        so_ = torch.empty(1, dtype=torch.float32, device=dev)
        ao_ = torch.empty(1, dtype=torch.float32, device=dev)
        reps = max(10, min(200, copies * 4))
        row = {}
        t = time_in_graph([lambda r, st: raw.check(L.fp8_quantize_blockwise(
            xs_[r % copies].data_ptr(), 1, R, C, 1, 128, 0, qs_[r % copies].data_ptr(), ss_[r % copies].data_ptr(),
            st), "1x128")], reps, dev)
        row["1x128_e4m3"] = round((3 * n + 4 * (n // 128)) / (t * 1e-3) / 1e9, 1)
        if R >= 128:
            t = time_in_graph([lambda r, st: raw.check(L.fp8_quantize_blockwise(
                xs_[r % copies].data_ptr(), 1, R, C, 128, 128, 0, qs_[r % copies].data_ptr(),
                st_[r % copies].data_ptr(), st), "128x128")], reps, dev)
            row["128x128_e4m3"] = round((3 * n + 4 * (n // 16384)) / (t * 1e-3) / 1e9, 1)
        # per-tensor: at least two inputs, so the reverse cast pass cannot hand the next launch's amax pass
        # its data in L2
        xp_ = xs_ if copies >= 2 else [x0, x0.clone()]
        t = time_in_graph([lambda r, st: raw.check(L.fp8_quantize_per_tensor(
            xp_[r % len(xp_)].data_ptr(), 1, n, 1, None, qs_[r % copies].data_ptr(), so_.data_ptr(),
            ao_.data_ptr(), st), "per-tensor")], reps, dev)
        row["per_tensor_current_e5m2"] = round(3 * n / (t * 1e-3) / 1e9, 1)
        t = time_in_graph([lambda r, st: raw.check(L.fp8_dequantize(
            qs_[r % copies].data_ptr(), 1, R, C, 0, 0, so_.data_ptr(), ys_[r % copies].data_ptr(), 1, st),
            "dequant")], reps, dev)
        row["per_tensor_dequant_bf16"] = round(3 * n / (t * 1e-3) / 1e9, 1)
        if R >= 128:
            for c_ in range(copies):  # every set's 128x128 codes and scales, untimed
                raw.check(L.fp8_quantize_blockwise(xs_[c_].data_ptr(), 1, R, C, 128, 128, 0, qs_[c_].data_ptr(),
                                                   st_[c_].data_ptr(), raw.stream), "128x128")
            t = time_in_graph([lambda r, st: raw.check(L.fp8_dequantize(
                qs_[r % copies].data_ptr(), 0, R, C, 128, 128, st_[r % copies].data_ptr(),
                ys_[r % copies].data_ptr(), 1, st), "dequant")], reps, dev)
            row["128x128_dequant_bf16"] = round((3 * n + 4 * (n // 16384)) / (t * 1e-3) / 1e9, 1)
        for c_ in range(copies):
            raw.check(L.fp8_quantize_blockwise(xs_[c_].data_ptr(), 1, R, C, 1, 128, 0, qs_[c_].data_ptr(),
                                               ss_[c_].data_ptr(), raw.stream), "1x128")
        t = time_in_graph([lambda r, st: raw.check(L.fp8_dequantize(
            qs_[r % copies].data_ptr(), 0, R, C, 1, 128, ss_[r % copies].data_ptr(), ys_[r % copies].data_ptr(), 1, st),
            "dequant")], reps, dev)
        row["1x128_dequant_bf16"] = round((3 * n + 4 * (n // 128)) / (t * 1e-3) / 1e9, 1)
        row["buffer_sets"] = copies
        sweep[f"2^{lg}"] = row
        del x0, xs_, xp_, qs_, ss_, st_, ys_
        torch.cuda.empty_cache()
    out["sweep_GB_s"] = sweep

    # per-tensor current scaling on small tensors (latency-bound): two passes vs the one-pass kernel, each
    # launch timed alone after an untimed L2 flush
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    st = stream.cuda_stream
    ws = torch.zeros(4, dtype=torch.int32, device=dev)
    so1 = torch.empty(1, dtype=torch.float32, device=dev)
    ao1 = torch.empty(1, dtype=torch.float32, device=dev)
    for key, label, x_small, dt, esz in (
            ("fp32_1MiB", "fp32 256x1024 outliers x1e4, seed 0 (the handbook's experiment tensor)",
             inputs.relerr_outlier_tensors()[1][1].to(dev), 0, 4),
            ("bf16_2^22", "bf16 randn 2^22 as [1024, 4096], 0.1% x1e3, seed 4", inputs.sweep_tensor(22, device=dev),
             1, 2)):
        nn = x_small.numel()
        qs_ = torch.empty(x_small.shape, dtype=torch.uint8, device=dev)
        two = lambda r: raw.check(L.fp8_quantize_per_tensor(x_small.data_ptr(), dt, nn, 0, None, qs_.data_ptr(),
                                                            so1.data_ptr(), ao1.data_ptr(), st), "per-tensor")
        one = lambda r: raw.check(L.fp8_quantize_per_tensor_fused(x_small.data_ptr(), dt, nn, 0, qs_.data_ptr(),
                                                                  so1.data_ptr(), ao1.data_ptr(), ws.data_ptr(), st),
                                  "fused per-tensor")
        t2, t1 = time_per_launch([two, one], 30, 5, stream, lambda: flush_buf.fill_(1))
        put(f"per_tensor_current_e4m3_{key}_two_pass", label + " (single call after an L2 flush)", (esz + 1) * nn, t2)
        put(f"per_tensor_current_e4m3_{key}_one_pass", label + " (single call after an L2 flush; cooperative "
            "one-pass kernel)", (esz + 1) * nn, t1)
        if key == "fp32_1MiB":
            # the handbook's experiment tensor in 1x128 blocks as well: quantize, then dequant back to fp32
            R1, C1 = x_small.shape
            sb_ = torch.empty(R1, C1 // 128, dtype=torch.float32, device=dev)
            yf_ = torch.empty(R1, C1, dtype=torch.float32, device=dev)
            bq = lambda r: raw.check(L.fp8_quantize_blockwise(x_small.data_ptr(), 0, R1, C1, 1, 128, 0,
                                                              qs_.data_ptr(), sb_.data_ptr(), st), "1x128")
            bd = lambda r: raw.check(L.fp8_dequantize(qs_.data_ptr(), 0, R1, C1, 1, 128, sb_.data_ptr(),
                                                      yf_.data_ptr(), 0, st), "dequant")
            tbq, tbd = time_per_launch([bq, bd], 30, 5, stream, lambda: flush_buf.fill_(1))
            nb1 = (esz + 1) * nn + 4 * (nn // 128)
            put("1x128_e4m3_fp32_1MiB", label + " (single call after an L2 flush)", nb1, tbq)
            put("1x128_dequant_fp32_1MiB", label + " (single call after an L2 flush)", nb1, tbd)
            del sb_, yf_
        del x_small, qs_
    del flush_buf
    out["note"] = ("large modes: back-to-back launches replayed from a CUDA graph, events around the replay; "
                   "frac is of the peak above")
    return out


def weight_roundtrip(dev, raw, peak, steps_list=(20, 2000)):
    """The bf16 4096x4096 weight (N(0, 0.02^2), seed 1): 128x128 E4M3 quantize + bf16 dequant per step.

    The 32 MiB weight fits in L2, so the steps rotate over enough buffer sets (x, codes, scales, output)
    that every step reads data last touched more than an L2's worth of traffic ago.  Each kernel moves
    48 MiB in under 10 us, so K steps are captured into one CUDA graph and timed with events around its
    replay.  Timed at several K: the replay's fixed cost (the graph launch before the first kernel and the
    drain after the last) is amortized over K, so K = 20 reads slower per step than K = 2000; the fit
    t(K) = t0 + K * t_step separates the two."""
    import torch
    from fine_grained_block_b200 import inputs
    L = raw.L
    R = C = 4096
    n = R * C
    qb = 3 * n + 4 * (n // 16384)
    per_set = n * (2 + 1 + 2) + 4 * 1024
    nsets = max(2, math.ceil(3 * L2_BYTES / per_set))
    w0 = inputs.weight_4096(seed=1).to(dev)
    xs = [w0] + [w0.clone() for _ in range(nsets - 1)]
    qs = [torch.empty(R, C, dtype=torch.uint8, device=dev) for _ in range(nsets)]
    ss = [torch.empty(R // 128, C // 128, dtype=torch.float32, device=dev) for _ in range(nsets)]
    ys = [torch.empty(R, C, dtype=torch.bfloat16, device=dev) for _ in range(nsets)]

    def fq(r, st):
        i = r % nsets
        raw.check(L.fp8_quantize_blockwise(xs[i].data_ptr(), 1, R, C, 128, 128, 0, qs[i].data_ptr(),
                                           ss[i].data_ptr(), st), "128x128")

    def fd(r, st):
        i = r % nsets
        raw.check(L.fp8_dequantize(qs[i].data_ptr(), 0, R, C, 128, 128, ss[i].data_ptr(), ys[i].data_ptr(), 1, st),
                  "dequant")

    out = {"workload": "bf16 weight 4096x4096 N(0,0.02^2), seed 1: 128x128 E4M3 quantize + bf16 dequant per step "
                       f"({nsets} rotating buffer sets, {nsets * per_set >> 20} MiB)", "by_steps": {}}
    fit = []
    for K in steps_list:
        ms = time_in_graph([fq, fd], K, dev) * K
        fit.append((K, ms))
        out["by_steps"][str(K)] = {"us_per_step": round(ms / K * 1e3, 3),
                                   "GB_s": round(2 * qb * K / (ms * 1e-3) / 1e9, 1),
                                   "frac_of_peak": round(2 * qb * K / (ms * 1e-3) / 1e9 / peak, 4)}
    (k0, m0), (k1, m1) = fit[0], fit[-1]
    t_step = (m1 - m0) / (k1 - k0)
    out["fit"] = {"us_per_step": round(t_step * 1e3, 3), "fixed_us_per_replay": round((m0 - k0 * t_step) * 1e3, 2),
                  "GB_s_per_step": round(2 * qb / (t_step * 1e-3) / 1e9, 1)}
    del xs, qs, ss, ys
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist
    from fine_grained_block_b200 import inputs

    world = env_int("WORLD_SIZE", 1)
    rank = env_int("RANK", 0)
    local = env_int("LOCAL_RANK", 0)
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    raw = Raw(stream)
    L, st = raw.L, raw.stream
    peak, peak_kind = measured_peaks()

    # the headline tensor, drawn on the host (rank 0's is the tensor the 2^30 parity test compares)
    x_cpu = inputs.sweep_tensor(LOG2_N, seed=4 + rank)
    assert tuple(x_cpu.shape) == (ROWS, COLS)
    qb, db = step_bytes()
    x = x_cpu.to(dev)
    q = torch.empty(ROWS, COLS, dtype=torch.uint8, device=dev)
    s = torch.empty(ROWS, COLS // 128, dtype=torch.float32, device=dev)
    y = torch.empty(ROWS, COLS, dtype=torch.bfloat16, device=dev)
    quant, deq = L.fp8_quantize_blockwise, L.fp8_dequantize

    def fq(bufs, stream_handle):
        xb, qb_, sb, _ = bufs
        raw.check(quant(xb.data_ptr(), 1, ROWS, COLS, *BLOCK, 0, qb_.data_ptr(), sb.data_ptr(), stream_handle),
                  "quantize")

    def fd(bufs, stream_handle):
        _, qb_, sb, yb = bufs
        raw.check(deq(qb_.data_ptr(), 0, ROWS, COLS, *BLOCK, sb.data_ptr(), yb.data_ptr(), 1, stream_handle),
                  "dequantize")

    main_set = (x, q, s, y)
    for _ in range(args.warmup):
        fq(main_set, st)
        fd(main_set, st)
    torch.cuda.synchronize()

    # The timed region: K steps launched eagerly, an event after every launch.  Each launch runs about
    # half a millisecond, so the host stays ahead of the device and the queue never drains.
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps + 1)]
    clocks = ClockSampler(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    evs[0].record(stream)
    for k in range(args.steps):
        fq(main_set, st)
        evs[2 * k + 1].record(stream)
        fd(main_set, st)
        evs[2 * k + 2].record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    if world > 1:
        dist.barrier()
    total_ms = evs[0].elapsed_time(evs[-1])
    tq = [evs[2 * k].elapsed_time(evs[2 * k + 1]) for k in range(args.steps)]
    td = [evs[2 * k + 1].elapsed_time(evs[2 * k + 2]) for k in range(args.steps)]
    tq_mean, td_mean = statistics.fmean(tq), statistics.fmean(td)
    stats = [total_ms, tq_mean, td_mean, statistics.median(tq), min(tq), statistics.median(td), min(td)]
    total_ms, tq_mean, td_mean, tq_med, tq_best, td_med, td_best = max_over_ranks(stats, world, device=dev)
    value = (qb + db) * args.steps * world / (total_ms * 1e-3) / 1e9

    # End to end through the same C ABI with host buffers: every step uploads its input from pinned host
    # memory, runs both kernels and downloads codes, scales and the dequantized tensor.  Upload, compute
    # and download run on three streams over two device buffer sets, ordered by events per set, so step
    # r's download (device -> host) overlaps step r+1's upload (host -> device).
    hx = x_cpu.pin_memory()
    hq = torch.empty(ROWS, COLS, dtype=torch.uint8).pin_memory()
    hs = torch.empty(ROWS, COLS // 128, dtype=torch.float32).pin_memory()
    hy = torch.empty(ROWS, COLS, dtype=torch.bfloat16).pin_memory()
    sets = [main_set, (torch.empty_like(x), torch.empty_like(q), torch.empty_like(s), torch.empty_like(y))]
    e2e_steps = max(3, min(args.steps, 10))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in sets]
    ev_comp = [torch.cuda.Event() for _ in sets]
    ev_out = [torch.cuda.Event() for _ in sets]
    used = [False] * len(sets)

    def e2e_step(r):
        i = r % len(sets)
        xb, qb_, sb, yb = sets[i]
        with torch.cuda.stream(s_in):
            if used[i]:
                s_in.wait_event(ev_comp[i])  # the previous use of this input buffer has been read
            xb.copy_(hx, non_blocking=True)
            ev_in[i].record(s_in)
        stream.wait_event(ev_in[i])
        if used[i]:
            stream.wait_event(ev_out[i])  # the previous results in this set have been downloaded
        fq(sets[i], st)
        fd(sets[i], st)
        ev_comp[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[i])
            hq.copy_(qb_, non_blocking=True)
            hs.copy_(sb, non_blocking=True)
            hy.copy_(yb, non_blocking=True)
            ev_out[i].record(s_out)
        used[i] = True

    for r in range(2):
        e2e_step(r)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(s_in)
    for r in range(e2e_steps):
        e2e_step(r)
    e1.record(s_out)
    torch.cuda.synchronize()
    (te,) = max_over_ranks([e0.elapsed_time(e1)], world, device=dev)
    e2e_value = (qb + db) * e2e_steps * world / (te * 1e-3) / 1e9

    # The link alone: the same uploads and downloads with no kernels, the two directions at once, as the
    # bound the e2e figure is read against.
    torch.cuda.synchronize()
    l0, l1, l_in = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                    torch.cuda.Event())
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    l0.record(s_in)
    s_out.wait_event(l0)
    for r in range(e2e_steps):
        xb, qb_, sb, yb = sets[r % len(sets)]
        with torch.cuda.stream(s_in):
            xb.copy_(hx, non_blocking=True)
        with torch.cuda.stream(s_out):
            hq.copy_(qb_, non_blocking=True)
            hs.copy_(sb, non_blocking=True)
            hy.copy_(yb, non_blocking=True)
    l_in.record(s_in)
    s_out.wait_event(l_in)
    l1.record(s_out)
    torch.cuda.synchronize()
    (tl,) = max_over_ranks([l0.elapsed_time(l1)], world, device=dev)
    link_value = (qb + db) * e2e_steps * world / (tl * 1e-3) / 1e9
    del sets, main_set, x, q, s, y, hq, hs, hy
    torch.cuda.empty_cache()

    line = None
    if rank == 0:
        def roofline(name, nbytes, ms_mean, ms_med, ms_best, share):
            achieved = nbytes / (ms_mean * 1e-3) / 1e9
            return {"bound": "hbm", "kernel": name, "achieved": round(achieved, 1), "peak": peak,
                    "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                    "traffic": committed_traffic(name), "alg_bytes_per_launch": nbytes,
                    "us_per_launch": round(ms_mean * 1e3, 2), "us_median": round(ms_med * 1e3, 2),
                    "us_best": round(ms_best * 1e3, 2), "share_of_step": round(share, 4)}
        share_q = tq_mean / (tq_mean + td_mean)
        # the roofline object is the dominant kernel's (the larger share of the step); the other follows
        rq = roofline("k_quant_rowblocks", qb, tq_mean, tq_med, tq_best, share_q)
        rd = roofline("k_dequant_flat", db, td_mean, td_med, td_best, 1 - share_q)
        dominant, second = (rd, rq) if td_mean >= tq_mean else (rq, rd)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "rows": ROWS, "cols": COLS, "block": list(BLOCK), "fmt": "e4m3",
                       "io": "bf16 -> e4m3 codes + fp32 scales -> bf16", "bytes_per_step": qb + db,
                       "l2": "inputs larger than L2 (2 GiB in, 1 GiB codes + 32 MiB scales, 2 GiB out per step); "
                             "no flush",
                       "parallelism": f"dp{world}: independent tensor per rank (seed 4+rank), no collective"},
            "roofline": dominant,
            "roofline_second_kernel": second,
            "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": hx.numel() * 2,
                    "d2h_bytes_per_step": ROWS * COLS + ROWS * (COLS // 128) * 4 + ROWS * COLS * 2,
                    "steps": e2e_steps,
                    "note": "pinned host buffers; uploads, kernels and downloads on three streams over two device "
                            "buffer sets, so one step's download overlaps the next step's upload",
                    "link_bound": {"value": round(link_value, 2), "unit": UNIT,
                                   "note": "the same uploads and downloads with no kernels, both directions at once"},
                    "frac_of_link_bound": round(e2e_value / link_value, 4)},
            "gpu_launches": 2 * args.steps,
            "timing": "K steps launched eagerly, an event after every launch; value = bytes / (last event - first)",
            "clocks": clocks.summary(),
        }
    bits = inputs.bf16_bits(x_cpu) if (world == 1 and rank == 0 and not args.no_cpu_baseline) else None
    del x_cpu, hx
    if world == 1 and not args.no_modes:
        line["modes"] = modes_breakdown(dev, stream, peak)
        line["modes"]["weight_4096_128x128_roundtrip"] = weight_roundtrip(dev, raw, peak)
    if bits is not None:
        line["cpu_baseline"] = cpu_baseline(bits)
        line["cpu_baseline_all_cores"] = cpu_baseline_all_cores(bits)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


KERNEL_PROBES = {
    "q128_weight4096": "k_quant_128x128: 128x128 E4M3 quantize of the bf16 weight 4096x4096",
    "dq128_weight4096": "k_dequant_128x128: its codes back to bf16",
    "fake_1x128_act": "k_fake_quant_1x128: 1x128 E4M3 round trip of the bf16 activations 16384x7168",
    "mx_act": "k_quant_rowblocks (Pow2Scale): MX 1x32 E4M3 quantize of the activations",
    "dqmx_act": "k_dequant_mx: those MX codes back to bf16",
    "cast_transpose_act": "k_tensor_cast_transpose: per-tensor E4M3 q and qt of the activations, delayed scale",
    "delayed_step_grads": "k_tensor_cast_delayed_step: one delayed E5M2 step (W 16) on the gradients 8192x8192",
    "delayed_step_grouped": "k_tensor_cast_delayed_step_grouped: 128 bf16 tensors of 2^20 in one call",
    "grouped_weights": "k_quant_grouped: 128 bf16 weights 1024x1024, 128x128 E4M3, in one call",
    "per_tensor_sweep28": "k_tensor_amax then k_tensor_cast: per-tensor current E5M2 of the sweep tensor 2^28",
}


def kernel_probe(args):
    """One launch of a named kernel on the workload its profile covers, between L2 cleaners (as in
    --traffic-probe), for an ncu capture; --probe-time K then times K single launches, each after an L2
    flush.  The workloads are those of `bench.py` modes, and small enough for a full ncu capture."""
    import torch
    from fine_grained_block_b200 import inputs
    from fine_grained_block_b200.binding import FP8BlockTensor, FP8DelayedTensor
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    raw = Raw(stream, args.lib)
    L, st = raw.L, raw.stream
    f32, u8, bf16 = torch.float32, torch.uint8, torch.bfloat16
    name = args.probe
    pre = []       # launches run once before the captured ones (the codes a dequant reads)
    launches = []  # (kernel, algorithmic bytes, fn(stream))
    keep = []      # tensors the launches use
    if name in ("q128_weight4096", "dq128_weight4096"):
        w = inputs.weight_4096(device=dev)
        R, C = w.shape
        n = w.numel()
        q = torch.empty(R, C, dtype=u8, device=dev)
        s = torch.empty(R // 128, C // 128, dtype=f32, device=dev)
        y = torch.empty(R, C, dtype=bf16, device=dev)
        quant = lambda s_: raw.check(L.fp8_quantize_blockwise(w.data_ptr(), 1, R, C, 128, 128, 0, q.data_ptr(),
                                                              s.data_ptr(), s_), "128x128")
        if name == "q128_weight4096":
            launches.append(("k_quant_128x128", 3 * n + 4 * (n // 16384), quant))
            outs = (q, s)
        else:
            pre.append(quant)
            launches.append(("k_dequant_128x128", 3 * n + 4 * (n // 16384), lambda s_: raw.check(L.fp8_dequantize(
                q.data_ptr(), 0, R, C, 128, 128, s.data_ptr(), y.data_ptr(), 1, s_), "dequant")))
            outs = (y,)
        keep += [w, q, s, y]
    elif name in ("fake_1x128_act", "mx_act", "dqmx_act", "cast_transpose_act"):
        a = inputs.activation_outlier_channels(device=dev)
        R, C = a.shape
        n = a.numel()
        q = torch.empty(R, C, dtype=u8, device=dev)
        y = torch.empty(R, C, dtype=bf16, device=dev)
        e8 = torch.empty(R, C // 32, dtype=u8, device=dev)
        qt = torch.empty(C, R, dtype=u8, device=dev)
        sc = torch.full((1,), 0.25, dtype=f32, device=dev)
        so = torch.empty(1, dtype=f32, device=dev)
        ao = torch.empty(1, dtype=f32, device=dev)
        mx = lambda s_: raw.check(L.fp8_quantize_mx(a.data_ptr(), 1, R, C, 0, 0, q.data_ptr(), e8.data_ptr(), s_), "mx")
        if name == "fake_1x128_act":
            launches.append(("k_fake_quant_1x128", 4 * n, lambda s_: raw.check(L.fp8_fake_quantize(
                a.data_ptr(), 1, R, C, 1, 128, 0, None, y.data_ptr(), None, s_), "fake quant")))
            outs = (y,)
        elif name == "mx_act":
            launches.append(("k_quant_rowblocks", 3 * n + n // 32, mx))
            outs = (q, e8)
        elif name == "dqmx_act":
            pre.append(mx)
            launches.append(("k_dequant_mx", 3 * n + n // 32, lambda s_: raw.check(L.fp8_dequantize_mx(
                q.data_ptr(), 0, R, C, e8.data_ptr(), y.data_ptr(), 1, s_), "mx dequant")))
            outs = (y,)
        else:
            launches.append(("k_tensor_cast_transpose", 4 * n, lambda s_: raw.check(
                L.fp8_quantize_per_tensor_transpose(a.data_ptr(), 1, R, C, 0, sc.data_ptr(), q.data_ptr(),
                                                    qt.data_ptr(), so.data_ptr(), ao.data_ptr(), s_), "transpose")))
            outs = (q, qt, ao)
        keep += [a, q, y, e8, qt, sc, so, ao]
    elif name == "delayed_step_grads":
        g = inputs.gradient_step(inputs.gradient_base(device=dev), 0)
        n = g.numel()
        q = torch.empty(g.shape, dtype=u8, device=dev)
        scale = torch.ones(1, dtype=f32, device=dev)
        hist = torch.zeros(16, dtype=f32, device=dev)
        state = torch.zeros(2, dtype=torch.int32, device=dev)
        used = torch.empty(1, dtype=f32, device=dev)
        amax = torch.empty(1, dtype=f32, device=dev)
        ws = torch.zeros(4, dtype=torch.int32, device=dev)
        launches.append(("k_tensor_cast_delayed_step", 3 * n, lambda s_: raw.check(L.fp8_quantize_delayed_step(
            g.data_ptr(), 1, n, 1, scale.data_ptr(), hist.data_ptr(), state.data_ptr(), 16, 0, 1.0, 1.0,
            q.data_ptr(), used.data_ptr(), amax.data_ptr(), ws.data_ptr(), s_), "delayed step")))
        outs = (q, amax)
        keep += [g, q, scale, hist, state, used, amax, ws]
    elif name == "delayed_step_grouped":
        gx = [inputs.random_matrix(1, 1 << 20, seed=300 + i, dtype=bf16, scale=1e-3, device=dev).reshape(-1)
              for i in range(128)]
        gq = [torch.empty(1 << 20, dtype=u8, device=dev) for _ in gx]
        gst = [(torch.ones(1, device=dev), torch.zeros(16, device=dev), torch.zeros(2, dtype=torch.int32, device=dev),
                torch.empty(1, device=dev), torch.empty(1, device=dev)) for _ in gx]
        gws = torch.zeros(len(gx) * 4, dtype=torch.int32, device=dev)
        garr = (FP8DelayedTensor * len(gx))(*[FP8DelayedTensor(x_.data_ptr(), q_.data_ptr(), x_.numel(), sc_.data_ptr(),
                                                                h_.data_ptr(), stt_.data_ptr(), su_.data_ptr(),
                                                                am_.data_ptr())
                                               for x_, q_, (sc_, h_, stt_, su_, am_) in zip(gx, gq, gst)])
        launches.append(("k_tensor_cast_delayed_step_grouped", 3 * sum(x_.numel() for x_ in gx), lambda s_: raw.check(
            L.fp8_quantize_delayed_step_grouped(garr, len(gx), 1, 1, 16, 0, 1.0, 1.0, gws.data_ptr(), s_),
            "grouped step")))
        outs = tuple(gq[:4])
        keep += [gx, gq, gst, gws, garr]
    elif name == "grouped_weights":
        ws_ = [inputs.random_matrix(1024, 1024, seed=100 + i, dtype=bf16, scale=0.02, device=dev) for i in range(128)]
        wq = [torch.empty(1024, 1024, dtype=u8, device=dev) for _ in ws_]
        wsc = [torch.empty(8, 8, dtype=f32, device=dev) for _ in ws_]
        arr = (FP8BlockTensor * len(ws_))(*[FP8BlockTensor(w.data_ptr(), q_.data_ptr(), s_.data_ptr(), 1024, 1024)
                                            for w, q_, s_ in zip(ws_, wq, wsc)])
        launches.append(("k_quant_grouped", sum(3 * w.numel() + 4 * 64 for w in ws_), lambda s_: raw.check(
            L.fp8_quantize_blockwise_grouped(arr, len(ws_), 1, 128, 128, 0, s_), "grouped")))
        outs = tuple(wq[:4]) + tuple(wsc[:4])
        keep += [ws_, wq, wsc, arr]
    else:  # per_tensor_sweep28
        x = inputs.sweep_tensor(28, device=dev)
        n = x.numel()
        q = torch.empty(x.shape, dtype=u8, device=dev)
        so = torch.empty(1, dtype=f32, device=dev)
        ao = torch.empty(1, dtype=f32, device=dev)
        launches.append(("k_tensor_amax + k_tensor_cast", 3 * n, lambda s_: raw.check(L.fp8_quantize_per_tensor(
            x.data_ptr(), 1, n, 1, None, q.data_ptr(), so.data_ptr(), ao.data_ptr(), s_), "per-tensor")))
        outs = (q, so, ao)
        keep += [x, q, so, ao]
    cleaner = torch.ones(1 << 28, dtype=bf16, device=dev)
    am = torch.empty(1, dtype=f32, device=dev)

    def clean():
        raw.check(L.fp8_amax(cleaner.data_ptr(), 1, cleaner.numel(), am.data_ptr(), st), "amax")

    for fn in pre:
        fn(st)
    clean()
    for _, _, fn in launches:
        fn(st)
        clean()
    torch.cuda.synchronize()
    same = None
    if args.lib:
        # a variant build must give the default build's bytes: rerun the default on copies of the outputs
        got = [t.clone() for t in outs]
        L_var, raw.L = raw.L, Raw(stream).L
        L = raw.L
        for fn in pre:
            fn(st)
        for _, _, fn in launches:
            fn(st)
        torch.cuda.synchronize()
        bits = lambda t: t.view(torch.int32) if t.dtype == f32 else t.view(torch.int16) if t.dtype == bf16 else t
        same = all(torch.equal(bits(g_), bits(o_)) for g_, o_ in zip(got, outs))
        raw.L = L = L_var
    out = {"probe": name, "what": KERNEL_PROBES[name], "lib": args.lib or "default", "same_as_default": same,
           "alg_bytes": {k: nb for k, nb, _ in launches}}
    if args.probe_time:
        for k, nb, fn in launches:
            (ms,) = time_per_launch([lambda r, fn=fn: fn(st)], args.probe_time, 3, stream, lambda: cleaner.fill_(1))
            out.setdefault("timing", {})[k] = {"us": round(ms * 1e3, 2), "GB_s": round(nb / (ms * 1e-3) / 1e9, 1),
                                               "note": "each launch alone after an L2 flush"}
    print(json.dumps({"kernel_probe": out}))
    return 0


def traffic_probe(args):
    """One launch of a kernel between L2 cleaners, for an ncu capture of DRAM bytes read and written.

    Sequence: cleaner, kernel, cleaner (and for the headline: quantize, cleaner, dequant, cleaner).  The
    cleaner is the library's amax kernel over a 512 MiB bf16 buffer: it reads more than the L2 holds and
    writes 4 bytes, so under `ncu --cache-control none` each probed kernel starts with none of its inputs
    in L2, and the dirty lines a kernel leaves in L2 are written back during the next cleaner, whose own
    DRAM writes are those write-backs alone.  A kernel's write traffic is therefore its own
    dram__bytes_write.sum plus that of the cleaner after it.

    --probe headline   the headline pair (1x128 quantize, dequant) on the 2^n sweep tensor;
    --probe 128x128    128x128 quantize of the 2^n sweep tensor;
    --probe bt1x128    1x128 quantize of x and x^T of the bf16 activations 16384x7168;
    --probe gemm_fwd / gemm_wgrad   the consumer GEMM (timing; its operands are quantized first);
    --probe gemm_4096               the forward GEMM at 4096 x 4096 x 4096;
    --probe gemm_wgrad_e4m3         the weight-gradient shape with both operands E4M3;
    --probe gemm_wgrad_b128         the weight-gradient shape with B in 128x128 blocks (the forward form);
    --probe gemm_wgrad_f32out       the weight-gradient GEMM writing fp32 instead of bf16;
    --probe per_tensor_1mib         per-tensor current scaling of the fp32 256x1024 experiment tensor in one
                                    pass (k_tensor_fused; --probe-time: each call timed alone after an L2
                                    flush, beside the two-pass path).
    --probe-time K     afterwards, also time K back-to-back launches of the probed kernel(s) (not under ncu).
    --lib PATH         use another build of the library (a variant built with tuning macros).
    The kernels of the other modes have probes of their own (KERNEL_PROBES, run by kernel_probe)."""
    import torch
    from fine_grained_block_b200 import inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    raw = Raw(stream, args.lib)
    L, st = raw.L, raw.stream
    if args.probe == "bt1x128":
        x = inputs.activation_outlier_channels(device=dev)
    elif args.probe == "per_tensor_1mib":
        x = inputs.relerr_outlier_tensors()[1][1].to(dev)
    elif args.probe.startswith("gemm"):
        # the consumer GEMM's operands, quantized by the library: forward (1x128 x 128x128, M N K =
        # 16384 4096 7168) or weight gradient (1x128 x 1x128, E5M2 x E4M3, 4096 7168 16384)
        wgrad = args.probe.startswith("gemm_wgrad")
        Mg, Ng, Kg = (4096, 7168, 16384) if wgrad else (4096, 4096, 4096) if args.probe == "gemm_4096" else \
            (16384, 4096, 7168)
        a_fmt = 1 if args.probe in ("gemm_wgrad", "gemm_wgrad_f32out") else 0  # gemm_wgrad_e4m3: both E4M3
        xa = inputs.random_matrix(Mg, Kg, seed=8 if wgrad else 6, dtype=torch.bfloat16, scale=1e-3 if wgrad else 1.0,
                                  outlier_frac=1e-3, factor=1e2, device=dev)
        xb = inputs.random_matrix(Ng, Kg, seed=9 if wgrad else 7, dtype=torch.bfloat16, scale=1.0 if wgrad else 0.02,
                                  outlier_frac=1e-3 if wgrad else 0.0, factor=1e2, device=dev)
        bro = 1 if wgrad and args.probe != "gemm_wgrad_b128" else 128  # gemm_wgrad_b128: B in 128x128 blocks
        qa = torch.empty(Mg, Kg, dtype=torch.uint8, device=dev)
        sa = torch.empty(Mg, Kg // 128, dtype=torch.float32, device=dev)
        qbm = torch.empty(Ng, Kg, dtype=torch.uint8, device=dev)
        sbm = torch.empty(Ng // bro, Kg // 128, dtype=torch.float32, device=dev)
        raw.check(L.fp8_quantize_blockwise(xa.data_ptr(), 1, Mg, Kg, 1, 128, a_fmt, qa.data_ptr(), sa.data_ptr(),
                                           st), "1x128")
        raw.check(L.fp8_quantize_blockwise(xb.data_ptr(), 1, Ng, Kg, bro, 128, 0, qbm.data_ptr(), sbm.data_ptr(), st),
                  "B")
        out_f32 = args.probe == "gemm_wgrad_f32out"  # the weight-gradient GEMM writing fp32
        x = torch.empty(Mg, Ng, dtype=torch.float32 if out_f32 else torch.bfloat16, device=dev)  # the GEMM's output
    else:
        x = inputs.sweep_tensor(args.traffic_log2n, seed=4, device=dev)
    R, C = x.shape
    n = x.numel()
    q = torch.empty(R, C, dtype=torch.uint8, device=dev)
    cleaner = torch.ones(1 << 28, dtype=torch.bfloat16, device=dev)
    am = torch.empty(1, dtype=torch.float32, device=dev)

    def clean():
        raw.check(L.fp8_amax(cleaner.data_ptr(), 1, cleaner.numel(), am.data_ptr(), st), "amax")

    launches = []
    if args.probe == "headline":
        s = torch.empty(R, C // 128, dtype=torch.float32, device=dev)
        y = torch.empty(R, C, dtype=torch.bfloat16, device=dev)
        qb, db = step_bytes(R, C)
        launches.append(("k_quant_rowblocks", qb, lambda stream_: raw.check(L.fp8_quantize_blockwise(
            x.data_ptr(), 1, R, C, *BLOCK, 0, q.data_ptr(), s.data_ptr(), stream_), "quantize")))
        launches.append(("k_dequant_flat", db, lambda stream_: raw.check(L.fp8_dequantize(
            q.data_ptr(), 0, R, C, *BLOCK, s.data_ptr(), y.data_ptr(), 1, stream_), "dequantize")))
    elif args.probe == "128x128":
        s = torch.empty(R // 128, C // 128, dtype=torch.float32, device=dev)
        launches.append(("k_quant_128x128", 3 * n + 4 * (n // 16384), lambda stream_: raw.check(
            L.fp8_quantize_blockwise(x.data_ptr(), 1, R, C, 128, 128, 0, q.data_ptr(), s.data_ptr(), stream_),
            "128x128")))
    elif args.probe == "per_tensor_1mib":
        s = torch.empty(1, dtype=torch.float32, device=dev)
        am1 = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.zeros(4, dtype=torch.int32, device=dev)
        launches.append(("k_tensor_fused", 5 * n, lambda stream_: raw.check(L.fp8_quantize_per_tensor_fused(
            x.data_ptr(), 0, n, 0, q.data_ptr(), s.data_ptr(), am1.data_ptr(), ws.data_ptr(), stream_),
            "fused per-tensor")))
    elif args.probe.startswith("gemm"):
        s = torch.empty(1, dtype=torch.float32, device=dev)
        flops = 2.0 * Mg * Ng * Kg
        launches.append(("k_gemm_blockwise", flops, lambda stream_: raw.check(L.fp8_gemm_blockwise_ex(
            qa.data_ptr(), sa.data_ptr(), a_fmt, qbm.data_ptr(), sbm.data_ptr(), bro, 0, Mg, Ng, Kg,
            x.data_ptr(), 0 if out_f32 else 1, stream_), "gemm")))
    else:
        s = torch.empty(R, C // 128, dtype=torch.float32, device=dev)
        qt = torch.empty(C, R, dtype=torch.uint8, device=dev)
        st_ = torch.empty(C, R // 128, dtype=torch.float32, device=dev)
        launches.append(("k_quant_block_transpose", 4 * n + 8 * (n // 128), lambda stream_: raw.check(
            L.fp8_quantize_blockwise_transpose(x.data_ptr(), 1, R, C, 1, 128, 0, q.data_ptr(), s.data_ptr(),
                                               qt.data_ptr(), st_.data_ptr(), stream_), "block transpose")))
    clean()
    for _, _, fn in launches:
        fn(st)
        clean()
    torch.cuda.synchronize()
    same = None
    if args.lib:
        # a variant build must give the default build's bytes: rerun the default on copies of the outputs
        outs = (q, s, qt, st_) if args.probe == "bt1x128" else (q, s)
        got = [t.clone() for t in outs]
        if args.probe.startswith("gemm"):  # the GEMM's result is within a bound, not bit-exact: compare loosely
            got[0] = x.clone()
        default = Raw(stream)
        L_var, raw.L = raw.L, default.L
        L = raw.L
        for _, _, fn in launches:
            fn(st)
        torch.cuda.synchronize()
        if args.probe.startswith("gemm"):
            same = bool(torch.allclose(got[0].float(), x.float(), rtol=2e-2, atol=1e-3 * float(x.float().abs().max())))
        else:
            same = all(torch.equal(g.view(torch.int32) if g.dtype == torch.float32 else g,
                                   o.view(torch.int32) if o.dtype == torch.float32 else o)
                       for g, o in zip(got, outs))
        raw.L = L = L_var
    out = {"probe": args.probe, "rows": R, "cols": C, "lib": args.lib or "default", "same_as_default": same,
           "alg_bytes": {name: nb for name, nb, _ in launches},
           "source_sha256": {k: source_hash(k) for k in KERNEL_SOURCES}}
    if args.probe_time and args.probe == "per_tensor_1mib":
        # a 1 MiB call is latency-bound: time each call alone after an L2 flush, beside the two-pass path
        two = lambda r: raw.check(L.fp8_quantize_per_tensor(x.data_ptr(), 0, n, 0, None, q.data_ptr(),
                                                            s.data_ptr(), am1.data_ptr(), st), "per-tensor")
        t_one, t_two = time_per_launch([lambda r: launches[0][2](st), two], args.probe_time, 5, stream,
                                       lambda: cleaner.fill_(1))
        out["timing"] = {"k_tensor_fused": {"us": round(t_one * 1e3, 2), "GB_s": round(5 * n / (t_one * 1e-3) / 1e9, 1)},
                         "two_pass": {"us": round(t_two * 1e3, 2), "GB_s": round(5 * n / (t_two * 1e-3) / 1e9, 1)},
                         "note": "each call timed alone after an L2 flush"}
    elif args.probe_time:
        del cleaner
        for name, nb, fn in launches:
            ms = time_in_graph([lambda r, stream_, fn=fn: fn(stream_)], args.probe_time, dev)
            rate = nb / (ms * 1e-3) / (1e12 if name == "k_gemm_blockwise" else 1e9)
            out.setdefault("timing", {})[name] = {"us": round(ms * 1e3, 2),
                                                  ("TFLOP_s" if name == "k_gemm_blockwise" else "GB_s"): round(rate, 1)}
    print(json.dumps({"traffic_probe": out}))
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-modes", action="store_true", help="skip the per-mode breakdown")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip timing the CPU oracle")
    ap.add_argument("--ref-budget-s", type=float, default=60.0,
                    help="reference arm: seconds of oracle work for warm-up + timed steps together")
    ap.add_argument("--traffic-probe", action="store_true",
                    help="run one launch of each headline kernel between L2 cleaners (for an ncu DRAM capture)")
    ap.add_argument("--traffic-log2n", type=int, default=LOG2_N, help="tensor size of --traffic-probe (2^n)")
    ap.add_argument("--probe", choices=["headline", "128x128", "bt1x128", "gemm_fwd", "gemm_wgrad", "gemm_wgrad_e4m3",
                                        "gemm_wgrad_b128", "gemm_wgrad_f32out", "gemm_4096", "per_tensor_1mib",
                                        *KERNEL_PROBES],
                    default="headline",
                    help="the kernel(s) of --traffic-probe")
    ap.add_argument("--probe-time", type=int, default=0, metavar="K",
                    help="with --traffic-probe: also time K graph-replayed launches of the probed kernel(s)")
    ap.add_argument("--lib", default=None, help="with --traffic-probe: a variant build of the library")
    ap.add_argument("--oracle-by-config", action="store_true",
                    help="time the CPU oracle on a sample of each configuration (host only)")
    ap.add_argument("--oracle-budget-s", type=float, default=1.5, help="seconds per leg of --oracle-by-config")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.oracle_by_config:
        return oracle_by_config(args)
    if args.traffic_probe and args.probe in KERNEL_PROBES:
        return kernel_probe(args)
    if args.traffic_probe:
        return traffic_probe(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
