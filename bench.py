#!/usr/bin/env python
"""Benchmark of the NVFP4 x Q8_0 kernels on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl nvq|reference]

Prints ONE JSON line on rank 0.  Default workload ``decode_sweep``: one step
quantises one token's activations (Q8_0) and runs the decode GEMV for each of
the four linear shapes of a 27B-class dense decoder, (K, N) = (5120, 5120),
(5120, 25600), (25600, 5120), (5120, 152064); the metric is weight GB/s
(NVFP4 weight bytes N*K*0.5625 streamed per second).  Other workloads:
``gemv_4096`` (M=1, K=N=4096), ``small_batch`` (M=2..16), ``prefill`` (GEMM,
M in {256, 2048}; metric TFLOP/s = 2*M*N*K/s), ``stack_decode`` and
``stack_prefill`` (all linears of a 64-layer dense decoder; tokens/s).

Timing: W untimed warm-up steps, then exactly K steps bracketed by a
barrier and a device synchronize, timed with CUDA events on the launching
stream; the time is the max over ranks.  The weights of one step exceed the
126 MB L2 (about 600 MB for the decode sweep), so no L2 flush is inserted.
The dominant kernel is additionally bracketed by its own events inside the
timed region for the roofline entry.  ``e2e`` repeats the K steps through the
same public entry points with each step's activations copied from pinned
host memory and its outputs copied back inside the timed region.

Multi-GPU (``torchrun --nproc-per-node N``): every rank runs the same
workload on its own GPU with no data exchange (independent replicas; the
only collectives are the timing barrier and max).  ``value`` is the units of
all ranks divided by the max time, ``scaling`` is "weak".

``--impl reference`` times the plain CPU oracle on the host cores (rank 0
only), each step a bounded sample of the same workload, on the same metric.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
WEIGHT_BYTES_PER_ELEMENT = 0.5625       # 4-bit code + one UE4M3 byte per 16


# ---------------------------------------------------------------------------
# process group, peaks, clocks
# ---------------------------------------------------------------------------

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend: str):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, value: float, device) -> float:
        """Max of a float over ranks (a timing reduction, not data)."""
        if self.pg is None:
            return value
        import torch
        t = torch.tensor([value], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": FALLBACK_BF16_TFLOPS, "source": "fallback"}


_REASON_FIELDS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms."""

    def __init__(self, device_index: int):
        self.samples = []
        self.proc = None
        self.thread = None
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.gpu = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:  # noqa: BLE001
            self.gpu = str(device_index)

    def start(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,"
             + ",".join("clocks_event_reasons." + r for r in _REASON_FIELDS))
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.gpu],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 3 + len(_REASON_FIELDS):
                continue
            try:
                sm, smax, pw = float(parts[0]), float(parts[1]), float(parts[2])
            except ValueError:
                continue
            active = [r for r, v in zip(_REASON_FIELDS, parts[3:]) if v.lower() == "active"]
            self.samples.append((time.time(), sm, smax, pw, active))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0: float, t1: float) -> dict:
        inside = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({r for s in inside for r in s[4]})
        return {"sm_mhz": statistics.median(s[1] for s in inside),
                "sm_max_mhz": max(s[2] for s in inside),
                "power_w_max": max(s[3] for s in inside),
                "reasons": reasons, "samples": len(inside)}


def source_hash(*names: str) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "bit_weight_quantized_nvq_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str, src_hash: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel on
    this workload, or None when absent or taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.txt")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"^source_hash:\s*(\S+)", text, re.M)
    m_bytes = re.search(r"^dram_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
    if not m_hash or not m_bytes or m_hash.group(1) != src_hash:
        return None
    return float(m_bytes.group(1))


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

class GemvWorkload:
    """M-token decode GEMVs over a list of (K, N) shapes; one step quantises
    each shape's activations and runs its GEMV."""

    kernel = "gemv"
    sources = ("gemv.cu", "nvq_device.cuh")

    def __init__(self, name, shapes, M, make_case):
        self.name, self.shapes, self.M, self.make_case = name, shapes, M, make_case
        self.metric = "nvfp4_q8_0_gemv_weight_GBps"
        self.unit = "GB/s"

    # --- setup -------------------------------------------------------------
    def setup(self, device):
        import torch
        from bit_weight_quantized_nvq_b200 import capi
        self.capi = capi
        self.layers = []
        for K, N in self.shapes:
            W, x = self.make_case(K, N)
            codes, scales, g = capi.pack_nvfp4(W)
            del W
            L = {"K": K, "N": N, "g": g,
                 "codes": torch.from_numpy(codes).to(device),
                 "scales": torch.from_numpy(scales).to(device),
                 "x": torch.from_numpy(x).to(device),
                 "x_host": torch.from_numpy(x).pin_memory(),
                 "q": torch.empty((self.M, K), dtype=torch.int8, device=device),
                 "d": torch.empty((self.M, K // 32), dtype=torch.float16, device=device),
                 "y": torch.empty((self.M, N), dtype=torch.float32, device=device)}
            L["y_host"] = torch.empty_like(L["y"], device="cpu").pin_memory()
            self.layers.append(L)

    def config(self):
        return {"workload": self.name, "M": self.M,
                "shapes_KN": [list(s) for s in self.shapes],
                "weights": "NVFP4 (E2M1 + UE4M3 per 16 + fp32 g), N(0,0.02^2)",
                "activations": "Q8_0 quantised per step on the GPU",
                "l2": "inputs larger than L2 (weights of one step %.0f MB > 126 MB)"
                      % (self.weight_bytes() / 1e6),
                "parallelism": "replicas"}

    def weight_bytes(self):
        return sum(N * K * WEIGHT_BYTES_PER_ELEMENT for K, N in self.shapes)

    def units_per_step(self):
        return self.weight_bytes() / 1e9          # GB

    def kernel_bytes(self, L):
        """Algorithmic bytes of one GEMV launch: weights + scales, the Q8_0
        activations and the fp32 output."""
        M, K, N = self.M, L["K"], L["N"]
        return N * K * WEIGHT_BYTES_PER_ELEMENT + M * K * (1 + 2 / 32) + 4 * M * N

    def launches_per_step(self):
        return 2 * len(self.layers)

    # --- one step ------------------------------------------------------------
    def step(self, stream, events=None, e2e=False):
        capi = self.capi
        for L in self.layers:
            if e2e:
                L["x"].copy_(L["x_host"], non_blocking=True)
            capi.quantize_act_q8_0(L["x"], L["q"], L["d"], stream=stream)
            if events is not None:
                ev0, ev1 = events.pop()
                ev0.record(stream)
            capi.gemv(L["codes"], L["scales"], L["g"], L["q"], L["d"], L["y"], stream=stream)
            if events is not None:
                ev1.record(stream)
                events.done.append((ev0, ev1, self.kernel_bytes(L)))
            if e2e:
                L["y_host"].copy_(L["y"], non_blocking=True)

    def e2e_bytes(self):
        h2d = sum(L["x"].numel() * 4 for L in self.layers)
        d2h = sum(L["y"].numel() * 4 for L in self.layers)
        return h2d, d2h

    # --- CPU oracle sample ---------------------------------------------------
    def oracle_prepare(self, rows_per_shape):
        import oracle as o
        self.o = o
        self.samples = []
        for K, N in self.shapes:
            W, x = self.make_case(K, N)
            g = o.nvfp4_tensor_scale(W)
            r = min(rows_per_shape, N)
            codes, scales, _ = o.pack_nvfp4(W[:r], g=g)
            del W
            self.samples.append((K, r, codes, scales, g, x))

    def oracle_step(self):
        """Quantise and dot the sampled rows; returns the sample's GB."""
        o = self.o
        gb = 0.0
        for K, r, codes, scales, g, x in self.samples:
            q, d = o.quantize_q8_0(x)
            o.dot_fp64(codes, scales, g, q, d)
            gb += r * K * WEIGHT_BYTES_PER_ELEMENT / 1e9
        return gb

    def oracle_sample_desc(self, rows):
        return (f"first {rows} rows of each of the {len(self.shapes)} shapes, "
                f"M={self.M}: oracle Q8_0 quantisation + fp64 dequantise-then-dot")


class EventPool:
    def __init__(self, n):
        import torch
        self.free = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                     for _ in range(n)]
        self.done = []

    def pop(self):
        return self.free.pop()


def make_workload(name: str):
    from bit_weight_quantized_nvq_b200 import workloads as wl
    if name == "decode_sweep":
        return GemvWorkload(name, wl.DECODE_SHAPES, 1, lambda K, N: wl.decode_case(K, N))
    if name == "gemv_4096":
        return GemvWorkload(name, [(4096, 4096)], 1, lambda K, N: wl.gemv_4096_case())
    if name.startswith("small_batch_m"):
        M = int(name[len("small_batch_m"):])
        return GemvWorkload(name, wl.SMALL_BATCH_SHAPES, M,
                            lambda K, N: wl.small_batch_case(M, K, N))
    raise SystemExit(f"unknown workload {name!r}")


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def run_nvq(args, dist: Dist):
    import torch
    torch.cuda.set_device(dist.local_rank)
    device = torch.device("cuda", dist.local_rank)
    dist.init("nccl")
    peaks = load_peaks()
    wk = make_workload(args.workload)
    wk.setup(device)
    stream = torch.cuda.current_stream(device)

    for _ in range(args.warmup):
        wk.step(stream)
    torch.cuda.synchronize()

    sampler = ClockSampler(dist.local_rank)
    sampler.start()
    time.sleep(0.3)
    nlaunch = len(wk.shapes) * args.steps
    events = EventPool(nlaunch)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start.record(stream)
    for _ in range(args.steps):
        wk.step(stream, events)
    end.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    dist.barrier()
    ms = start.elapsed_time(end)
    kernel_ms = sum(a.elapsed_time(b) for a, b, _ in events.done)
    kernel_bytes = sum(nb for _, _, nb in events.done)
    n_kernel = len(events.done)
    time.sleep(0.2)
    sampler.stop()
    clocks = sampler.summary(t_wall0 - 0.15, t_wall1 + 0.15)

    # e2e: the same K steps with host<->device copies inside the timed region
    for _ in range(max(1, args.warmup // 2)):
        wk.step(stream, e2e=True)
    torch.cuda.synchronize()
    dist.barrier()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for _ in range(args.steps):
        wk.step(stream, e2e=True)
    e_end.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    e2e_ms = e_start.elapsed_time(e_end)

    ms_max = dist.max(ms, device)
    e2e_ms_max = dist.max(e2e_ms, device)
    units = wk.units_per_step() * args.steps * dist.world
    value = units / (ms_max / 1e3)
    e2e_value = units / (e2e_ms_max / 1e3)

    achieved = kernel_bytes / (kernel_ms / 1e3) / 1e9       # GB/s
    src_hash = source_hash(*wk.sources)
    traffic = profiled_traffic(wk.kernel, wk.name, src_hash)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic,
                "algorithmic_bytes_per_launch": kernel_bytes / max(1, n_kernel),
                "kernel": wk.kernel, "launches": n_kernel,
                "avg_launch_us": round(kernel_ms * 1e3 / max(1, n_kernel), 3),
                "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs, copy)"}

    cpu = None
    if dist.rank == 0 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wk, args.cpu_seconds)

    h2d, d2h = wk.e2e_bytes()
    line = {
        "metric": wk.metric, "value": round(value, 2), "unit": wk.unit,
        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 x q8_0 (int32 subblock sums, fp32 accumulate)",
        "data": "synthetic (seeded; shapes and distributions of the workload)",
        "config": wk.config(),
        "impl": "nvq",
        "e2e": {"value": round(e2e_value, 2), "unit": wk.unit,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": wk.launches_per_step() * args.steps,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "clocks": clocks,
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


def cpu_baseline(wk, seconds: float):
    """The oracle, timed on the host on a bounded sample of the workload."""
    import threadpoolctl
    rows = 64
    wk.oracle_prepare(rows)
    with threadpoolctl.threadpool_limits(1):
        t0 = time.perf_counter()
        wk.oracle_step()
        t_small = time.perf_counter() - t0
        rows = int(max(64, min(8192, rows * seconds / max(t_small, 1e-3))))
        wk.oracle_prepare(rows)
        t0 = time.perf_counter()
        gb = wk.oracle_step()
        t = time.perf_counter() - t0
    return {"value": round(gb / t, 4), "unit": wk.unit, "cores": 1, "kind": "oracle",
            "sample": wk.oracle_sample_desc(rows), "seconds": round(t, 2)}


def run_reference(args, dist: Dist):
    """The oracle as the reference arm: rank 0 only, on the host cores."""
    if dist.rank != 0:
        return
    import threadpoolctl
    wk = make_workload(args.workload)
    # size the per-step sample so that warm-up + timed steps take about
    # --cpu-seconds * 6 in total (a few minutes at most)
    budget = 6 * args.cpu_seconds / (args.steps + args.warmup)
    rows = 64
    wk.oracle_prepare(rows)
    with threadpoolctl.threadpool_limits(1):
        t0 = time.perf_counter()
        wk.oracle_step()
        t_small = time.perf_counter() - t0
    rows = int(max(8, min(8192, rows * budget / max(t_small, 1e-4))))
    wk.oracle_prepare(rows)
    with threadpoolctl.threadpool_limits(1):
        for _ in range(args.warmup):
            wk.oracle_step()
        t0 = time.perf_counter()
        gb = 0.0
        for _ in range(args.steps):
            gb += wk.oracle_step()
        t = time.perf_counter() - t0
    value = gb / t
    desc = wk.oracle_sample_desc(rows)
    line = {
        "metric": wk.metric, "value": round(value, 4), "unit": wk.unit,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 (int64 subblock sums)",
        "data": "synthetic (seeded; a bounded row sample of the workload)",
        "config": wk.config() if hasattr(wk, "config") else {"workload": args.workload},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": wk.unit, "cores": 1,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 4), "unit": wk.unit,
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="decode_sweep")
    ap.add_argument("--impl", choices=["nvq", "reference"], default="nvq")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target duration of the oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
    else:
        run_nvq(args, dist)


if __name__ == "__main__":
    main()
