#!/usr/bin/env python
"""Benchmark of the NVFP4 x Q8_0 kernels on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl nvq|reference] [--no-sub]

Prints ONE JSON line on rank 0.

Workloads (``--workload``; the line's headline is this one, default
``decode_sweep``, and unless ``--no-sub`` the line also carries every other
workload under ``"workloads"``, each measured the same way):
  decode_sweep            one step quantises one token's activations (Q8_0)
                          and runs the decode GEMV for each of the four
                          linear shapes of a 27B-class dense decoder,
                          (K, N) = (5120, 5120), (5120, 25600), (25600, 5120),
                          (5120, 152064).  Metric: weight GB/s (NVFP4 weight
                          bytes N*K*0.5625 streamed per second).
  gemv_4096               M=1, K=N=4096.
  small_batch_m{2,4,8,16} M tokens, (5120, 25600), (25600, 5120), through
                          nvq_gemm (its small-token tensor-core schedule).
  prefill_m{256,2048}     Q8_0 + tcgen05 GEMM over (5120, 5120), (5120, 25600),
                          (25600, 5120).  Metric: algorithmic TFLOP/s 2*M*N*K.
  stack_decode            all 448 linears of a 64-layer dense decoder (17.9 GB
                          of NVFP4 weights resident), one token.  Metric:
                          tokens/s of the linear layers.
  stack_prefill           the same stack for 2048 tokens.
  w4a16_decode            the decode-sweep shapes at one token with fp16
                          activations (nvq_gemm_w4a16).  Metric: weight GB/s.
  nvf4_prefill_m{256,2048} NVFP4 activations (nvq_quantize_act_nvfp4) and the
                          block-scaled FP4 tensor-core GEMM (nvq_gemm_nvf4)
                          over the prefill shapes.  Metric: TFLOP/s 2*M*N*K,
                          against the FP4 dense peak (measured bf16 x 4, the
                          nominal FP4/bf16 ratio).
  moe_decode              mixture-of-experts decode (mul_mat_id): 16 tokens,
                          each times 6 of 256 experts (K = 2048, N = 1536),
                          a different seeded routing every step.  Metric:
                          weight GB/s of the selected experts' rows.

Timing: W untimed eager warm-up steps; the K timed steps are captured once
into a CUDA graph (the public entry points only enqueue work) and replayed
inside the timed region, bracketed by a barrier and a device synchronize and
timed with CUDA events on the launching stream; the time is the max over
ranks.  One step's inputs exceed the 126 MB L2 in every workload (600 MB of
weights for the decode sweep), so no L2 flush is inserted.

Roofline of the dominant kernel (``roofline``): for the GEMV and GEMM
workloads each shape's dominant launch (nvq_gemv; nvq_gemm) is timed alone in
its own event-free CUDA graph of back-to-back launches that rotate through
enough copies of the weights (at least 4x the L2 size) that no launch finds
its weights in L2; achieved = algorithmic bytes (or flops) of one launch of
every shape / the sum of their launch times, with the per-shape rates
listed.  ``step_achieved`` divides the same amount by the whole step (which
also holds the quantiser launches).  For the stack the unit is the whole
pass (its launches are the step).

``e2e`` runs the same K steps through the public Python API eagerly, with each
step's activations copied from pinned host memory and its outputs copied back
inside the timed region (the weights are resident model parameters).

``cpu_baseline`` times the plain CPU oracle on a bounded sample of the same
workload: on one host core, and (``all_cores``) spread over every core of the
host in a pool of spawned worker processes, one numpy thread each.

Multi-GPU (``torchrun --nproc-per-node N``): every rank runs the same
workload on its own GPU with no data exchange (independent replicas; the
only collectives are the timing barrier and max).  ``value`` is the units of
all ranks divided by the max time; ``scaling`` is "weak".

``--impl reference`` times the plain CPU oracle on the host cores (rank 0
only), each step a bounded sample of the same workload, on the same metric.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
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
L2_BYTES = 126e6
SUB_WORKLOADS = ["gemv_4096", "small_batch_m2", "small_batch_m4", "small_batch_m8",
                 "small_batch_m16", "prefill_m256", "prefill_m2048", "stack_decode",
                 "stack_prefill", "moe_decode", "w4a16_decode", "nvf4_prefill_m2048"]


# ---------------------------------------------------------------------------
# process group, peaks, clocks, profiles
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
    """nvidia-smi SM clocks, power and throttle reasons every 100 ms."""

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
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed region"
        if not inside:
            # the timed region was shorter than one sample: the nearest ones
            near = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
            inside, window = near, "nearest samples (timed region shorter than one sample)"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({r for s in inside for r in s[4]})
        return {"sm_mhz": statistics.median(s[1] for s in inside),
                "sm_max_mhz": max(s[2] for s in inside),
                "power_w_max": max(s[3] for s in inside),
                "reasons": reasons, "samples": len(inside), "window": window}


def source_hash(*names: str) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "bit_weight_quantized_nvq_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str, src_hash: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel on
    this workload, or None when absent or taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"^source_hash:\s*(\S+)", text, re.M)
    m_bytes = re.search(r"^dram_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
    if not m_hash or not m_bytes or m_hash.group(1) != src_hash:
        return None
    return float(m_bytes.group(1))


def gemm_launches(M: int, N: int, K: int) -> int:
    """Kernels nvq_gemm launches after the Q8_0 expansion for M > 16 tokens:
    the persistent tcgen05 GEMM, plus the fix-up of its stream-K tiles when
    the tiles (128 tokens x 256 weight rows) do not divide evenly over the
    CTA pairs (one pair per two SMs)."""
    import torch
    pairs = torch.cuda.get_device_properties(0).multi_processor_count // 2
    tiles = -(-M // 128) * -(-(-(-N // 128)) // 2)
    stages = -(-K // 128)
    P = min(pairs, tiles * stages)
    return 1 + (1 if tiles % P else 0)


def replay_ms(graph, stream) -> float:
    """Device time of one replay of a captured graph (CUDA events on the
    launching stream, synchronised on both sides)."""
    import torch
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    graph.replay()
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end)


def l2_copies(nbytes: float) -> int:
    """Weight copies to rotate through so that a launch never finds its
    weights in L2 (at least 4x L2 in total, at least 2)."""
    return max(2, math.ceil(4 * L2_BYTES / max(nbytes, 1.0)))


# ---------------------------------------------------------------------------
# oracle tasks (CPU baseline): quantise a row sample's activations and take
# the fp64 dequantise-then-dot of a block of weight rows
# ---------------------------------------------------------------------------

def oracle_task(task):
    """Run one oracle task, (codes, scales, g, x, reps, units) -> units: the
    oracle's Q8_0 quantisation of x, then its fp64 dequantise-then-dot of the
    weight block, `reps` times (x given as fp16 bit patterns, uint16: the
    fp16-activation dot instead; x = ("nvf4", fp32 x): the oracle's NVFP4
    activation quantiser and the NVFP4 x NVFP4 dot)."""
    import oracle as o
    codes, scales, g, x, reps, units = task
    if isinstance(x, tuple):              # ("nvf4", fp32 x): NVFP4 activations
        ac, as_, ag = o.quantize_act_nvfp4(x[1])
        for _ in range(reps):
            o.dot_fp64_nvf4(codes, scales, g, ac, as_, ag)
        return units
    if x.dtype == np.uint16:
        for _ in range(reps):
            o.dot_fp64_f16(codes, scales, g, x)
        return units
    q, d = o.quantize_q8_0(x)
    for _ in range(reps):
        o.dot_fp64(codes, scales, g, q, d)
    return units


def _pool_init():
    import oracle  # noqa: F401  (imported once per worker, outside the timing)


def _noop(_):
    return 0


def split_tasks(tasks, parts: int):
    """Split every task's repetitions into about `parts` tasks (units in
    proportion)."""
    out = []
    for codes, scales, g, x, reps, units in tasks:
        k = max(1, min(parts, reps))
        bounds = np.linspace(0, reps, k + 1).astype(int)
        for a, b in zip(bounds[:-1], bounds[1:]):
            if b > a:
                out.append((codes, scales, g, x, int(b - a), units * (b - a) / reps))
    return out


class OraclePool:
    """Worker processes (spawned, one numpy thread each) over all host cores."""

    def __init__(self):
        import concurrent.futures as cf
        import multiprocessing as mp
        try:
            self.cores = len(os.sched_getaffinity(0))
        except AttributeError:
            self.cores = os.cpu_count() or 1
        self.cores = max(1, min(self.cores, 128))
        saved = {k: os.environ.get(k) for k in
                 ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        for k in saved:
            os.environ[k] = "1"
        try:
            self.ex = cf.ProcessPoolExecutor(self.cores, mp_context=mp.get_context("spawn"),
                                             initializer=_pool_init)
            list(self.ex.map(_noop, range(self.cores * 2)))   # start every worker
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v

    def run(self, tasks) -> float:
        parts = split_tasks(tasks, self.cores)
        return float(sum(self.ex.map(oracle_task, parts)))

    def close(self):
        self.ex.shutdown(wait=True, cancel_futures=True)


def run_tasks_serial(tasks) -> float:
    return float(sum(oracle_task(t) for t in tasks))


# The oracle packs a small base block of each matrix's rows once (its packer
# is far slower than its dot product); a sample of any size runs the oracle's
# dot over that block repeatedly.  The dot costs the same whatever the values.
ORACLE_BASE_ROWS = 64
_ORACLE_BASE = {}


def oracle_base(key, make):
    """(codes, scales, g, x) of a base block, packed by the oracle, cached."""
    if key not in _ORACLE_BASE:
        import oracle as o
        W, x = make()
        codes, scales, g = o.pack_nvfp4(W)
        _ORACLE_BASE[key] = (codes, scales, g, x)
    return _ORACLE_BASE[key]


def sample_task(base, rows: int, units_per_row: float):
    """A task that runs the oracle over `rows` weight rows as repetitions of
    the base block (rows rounded up to whole blocks)."""
    codes, scales, g, x = base
    reps = max(1, -(-rows // codes.shape[0]))
    return (codes, scales, g, x, reps, units_per_row * reps * codes.shape[0])


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

class GemvWorkload:
    """M-token decode GEMVs over a list of (K, N) shapes; one step quantises
    each shape's activations and runs its GEMV."""

    kernel = "gemv"
    sources = ("gemv.cu", "nvq_device.cuh", "tcgen05.cuh")
    bound = "hbm"
    dtype = "nvfp4 x q8_0 (int32 subblock sums, fp32 accumulate)"
    metric = "nvfp4_q8_0_gemv_weight_GBps"
    unit = "GB/s"

    def __init__(self, name, shapes, M, make_case, oracle_rows):
        self.name, self.shapes, self.M = name, shapes, M
        self.make_case, self.oracle_rows = make_case, oracle_rows

    def setup(self, device):
        import torch
        from bit_weight_quantized_nvq_b200 import capi
        self.capi = capi
        self.cases = []
        for K, N in self.shapes:
            W, x = self.make_case(K, N)
            codes, scales, g = capi.pack_nvfp4(W)
            del W
            c = {"K": K, "N": N, "g": g,
                 "codes": torch.from_numpy(codes).to(device),
                 "scales": torch.from_numpy(scales).to(device),
                 "x": torch.from_numpy(x).to(device),
                 "x_host": torch.from_numpy(x).pin_memory(),
                 "q": torch.empty((self.M, K), dtype=torch.int8, device=device),
                 "d": torch.empty((self.M, K // 32), dtype=torch.float16, device=device),
                 "y": torch.empty((self.M, N), dtype=torch.float32, device=device)}
            c["y_host"] = torch.empty((self.M, N), dtype=torch.float32).pin_memory()
            self.cases.append(c)

    def config(self):
        return {"workload": self.name, "M": self.M,
                "shapes_KN": [list(s) for s in self.shapes],
                "weights": "NVFP4 (E2M1 + UE4M3 per 16 + fp32 g), N(0,0.02^2)",
                "activations": "fp32 -> Q8_0 on the GPU every step (nvq_quantize_act_q8_0)",
                "l2": "inputs larger than L2 (weights of one step %.0f MB > 126 MB)"
                      % (self.weight_bytes() / 1e6),
                "parallelism": "replicas"}

    def weight_bytes(self):
        return sum(N * K * WEIGHT_BYTES_PER_ELEMENT for K, N in self.shapes)

    def units_per_step(self):
        return self.weight_bytes() / 1e9          # GB

    def kernel_amount(self, K, N):
        """Algorithmic bytes of one GEMV launch: NVFP4 weights, the Q8_0
        activations and the fp32 output."""
        M = self.M
        return N * K * WEIGHT_BYTES_PER_ELEMENT + M * K * (1 + 2 / 32) + 4 * M * N

    def launches_per_step(self):
        return 2 * len(self.cases)

    def dominant(self, c, codes, scales, stream):
        self.capi.gemv(codes, scales, c["g"], c["q"], c["d"], c["y"], stream=stream)

    def step(self, stream, e2e=False):
        capi = self.capi
        for c in self.cases:
            if e2e:
                c["x"].copy_(c["x_host"], non_blocking=True)
            capi.quantize_act_q8_0(c["x"], c["q"], c["d"], stream=stream)
            self.dominant(c, c["codes"], c["scales"], stream)
            if e2e:
                c["y_host"].copy_(c["y"], non_blocking=True)

    def e2e_bytes(self):
        return (sum(c["x"].numel() * 4 for c in self.cases),
                sum(c["y"].numel() * 4 for c in self.cases))

    def shape_timings(self, stream, reps):
        """Per shape: the dominant launch alone, back to back in an event-free
        graph, rotating through weight copies that defeat L2."""
        import torch
        out = []
        for c in self.cases:
            K, N = c["K"], c["N"]
            ncopy = l2_copies(N * K * WEIGHT_BYTES_PER_ELEMENT)
            copies = [(c["codes"], c["scales"])] + [
                (c["codes"].clone(), c["scales"].clone()) for _ in range(ncopy - 1)]
            for cc, ss in copies[:2]:
                self.dominant(c, cc, ss, stream)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                s = torch.cuda.current_stream()
                for i in range(reps):
                    cc, ss = copies[i % ncopy]
                    self.dominant(c, cc, ss, s)
            graph.replay()
            ms = replay_ms(graph, stream)
            del graph, copies
            torch.cuda.empty_cache()
            out.append({"K": K, "N": N, "us_per_launch": ms * 1e3 / reps,
                        "amount": self.kernel_amount(K, N), "weight_copies": ncopy})
        return out

    # --- CPU oracle sample ---------------------------------------------------
    def oracle_tasks(self, rows):
        tasks = []
        for K, N in self.shapes:
            base = oracle_base(("gemv", self.name, K, N),
                               lambda: self.oracle_rows(K, N, ORACLE_BASE_ROWS))
            tasks.append(sample_task(base, rows, K * WEIGHT_BYTES_PER_ELEMENT / 1e9))
        return tasks

    def oracle_sample_desc(self, rows):
        return (f"{rows} weight rows of each of the {len(self.shapes)} shapes (the first "
                f"{ORACLE_BASE_ROWS} rows, oracle-packed, run repeatedly), M={self.M}: oracle Q8_0 "
                "quantisation + fp64 dequantise-then-dot")


class SmallGemmWorkload(GemvWorkload):
    """Small-batch decode: Q8_0 of M <= 16 tokens and nvq_gemm, which runs
    the small-token tensor-core schedule; metric as the GEMV (weight GB/s)."""

    kernel = "gemm_small"
    sources = ("gemm_small.cu", "nvq_device.cuh", "tcgen05.cuh")   # the dominant kernel's code
    dtype = "nvfp4 x q8_0 (exact fp16 operands, fp32 accumulate)"

    def setup(self, device):
        import torch
        super().setup(device)
        for c in self.cases:
            c["ws"] = torch.empty(self.capi.gemm_workspace_size(self.M, c["N"], c["K"]),
                                  dtype=torch.uint8, device=device)

    def config(self):
        cfg = super().config()
        cfg["path"] = "nvq_gemm small-token tcgen05 schedule"
        return cfg

    def launches_per_step(self):
        # quantise, expand, tcgen05 kernel, and the fixed-order sum of split tiles
        return 4 * len(self.cases)

    def dominant(self, c, codes, scales, stream):
        self.capi.gemm(codes, scales, c["g"], c["q"], c["d"], c["y"], c["ws"], stream=stream)


class GemmWorkload(GemvWorkload):
    """Prefill: Q8_0 of M tokens and the tcgen05 GEMM for each shape."""

    kernel = "gemm"
    sources = ("gemm_tcgen05.cu", "nvq_device.cuh", "tcgen05.cuh")
    bound = "tensor"
    dtype = "nvfp4 x q8_0 (exact fp16 operands, fp32 accumulate)"
    metric = "nvfp4_q8_0_prefill_gemm_TFLOPs"
    unit = "TFLOP/s"

    def __init__(self, name, shapes, M):
        from bit_weight_quantized_nvq_b200 import workloads as wl
        super().__init__(name, shapes, M, lambda K, N: wl.prefill_case(M, K, N), None)

    def setup(self, device):
        import torch
        super().setup(device)
        for c in self.cases:
            c["ws"] = torch.empty(self.capi.gemm_workspace_size(self.M, c["N"], c["K"]),
                                  dtype=torch.uint8, device=device)

    def config(self):
        return {"workload": self.name, "M": self.M,
                "shapes_KN": [list(s) for s in self.shapes],
                "weights": "NVFP4, N(0,0.02^2)",
                "activations": "fp32 N(0,1), 0.1% channels x50 -> Q8_0 on the GPU every step",
                "l2": "inputs larger than L2 (activations and weights of one step > 126 MB)",
                "parallelism": "replicas"}

    def units_per_step(self):
        return sum(2.0 * self.M * N * K for K, N in self.shapes) / 1e12   # TFLOP

    def kernel_amount(self, K, N):
        return 2.0 * self.M * N * K

    def launches_per_step(self):
        # quantise, expand, tcgen05 GEMM (and the fix-up of its stream-K tiles)
        return sum(2 + gemm_launches(self.M, c["N"], c["K"]) for c in self.cases)

    def dominant(self, c, codes, scales, stream):
        self.capi.gemm(codes, scales, c["g"], c["q"], c["d"], c["y"], c["ws"], stream=stream)

    def oracle_tasks(self, rows):
        from bit_weight_quantized_nvq_b200 import workloads as wl
        toks = max(1, min(self.M, 16))
        tasks = []
        for K, N in self.shapes:
            base = oracle_base(
                ("gemm", self.name, K, N),
                lambda: (wl.weight_rows("prefill", "W", N, K, ORACLE_BASE_ROWS),
                         wl.activations("prefill", "x", self.M, K, "normal",
                                        outliers=True)[:toks]))
            tasks.append(sample_task(base, rows, 2.0 * toks * K / 1e12))
        return tasks

    def oracle_sample_desc(self, rows):
        toks = max(1, min(self.M, 16))
        return (f"{toks} tokens x {rows} weight rows of each of the {len(self.shapes)} shapes "
                f"(the first {ORACLE_BASE_ROWS} rows, oracle-packed, run repeatedly): oracle Q8_0 + "
                "fp64 dequantise-then-dot")


class Nvf4GemmWorkload(GemmWorkload):
    """Prefill on the block-scaled FP4 path: NVFP4 quantisation of M tokens
    (nvq_quantize_act_nvfp4) and nvq_gemm_nvf4 for each shape."""

    kernel = "gemm_nvf4"
    sources = ("nvf4.cu", "tcgen05.cuh")
    dtype = "nvfp4 x nvfp4 (block-scaled e2m1 tensor-core products, fp32 accumulate)"
    metric = "nvfp4_nvfp4_prefill_gemm_TFLOPs"
    peak_scale = 4.0
    peak_note = "bf16_tflops (burst) x 4, the nominal dense FP4/bf16 ratio (9 / 2.25 PFLOP/s)"

    def setup(self, device):
        import torch
        GemvWorkload.setup(self, device)
        for c in self.cases:
            M, K = self.M, c["K"]
            c["ac"] = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
            c["as"] = torch.empty((M, K // 16), dtype=torch.uint8, device=device)
            c["ag"] = torch.empty((M,), dtype=torch.float32, device=device)
            del c["q"], c["d"]
            self.capi.quantize_act_nvfp4(c["x"])      # library warm (tensor maps, attributes)

    def config(self):
        cfg = super().config()
        cfg["activations"] = ("fp32 N(0,1), 0.1% channels x50 -> NVFP4 (per-token fp32 scale) "
                              "on the GPU every step")
        cfg["path"] = "nvq_quantize_act_nvfp4 + nvq_gemm_nvf4 (tcgen05.mma kind::mxf4nvf4)"
        return cfg

    def launches_per_step(self):
        return 2 * len(self.cases)       # quantise, block-scaled GEMM

    def quantize(self, c, stream):
        lib = self.capi.lib()
        st = lib.nvq_quantize_act_nvfp4(c["x"].data_ptr(), self.M, c["K"], c["ac"].data_ptr(),
                                        c["as"].data_ptr(), c["ag"].data_ptr(), stream.cuda_stream)
        if st != 0:
            raise self.capi.NVQError("nvq_quantize_act_nvfp4", st)

    def dominant(self, c, codes, scales, stream):
        self.capi.gemm_nvf4(codes, scales, c["g"], c["ac"], c["as"], c["ag"], c["y"],
                            stream=stream)

    def step(self, stream, e2e=False):
        for c in self.cases:
            if e2e:
                c["x"].copy_(c["x_host"], non_blocking=True)
            self.quantize(c, stream)
            self.dominant(c, c["codes"], c["scales"], stream)
            if e2e:
                c["y_host"].copy_(c["y"], non_blocking=True)

    def oracle_tasks(self, rows):
        from bit_weight_quantized_nvq_b200 import workloads as wl
        toks = max(1, min(self.M, 16))
        tasks = []
        for K, N in self.shapes:
            base = oracle_base(
                ("gemm", self.name, K, N),
                lambda K=K, N=N: (wl.weight_rows("prefill", "W", N, K, ORACLE_BASE_ROWS),
                                  wl.activations("prefill", "x", self.M, K, "normal",
                                                 outliers=True)[:toks]))
            codes, scales, g, x = base
            tasks.append(sample_task((codes, scales, g, ("nvf4", x)), rows,
                                     2.0 * toks * K / 1e12))
        return tasks

    def oracle_sample_desc(self, rows):
        toks = max(1, min(self.M, 16))
        return (f"{toks} tokens x {rows} weight rows of each of the {len(self.shapes)} shapes "
                f"(the first {ORACLE_BASE_ROWS} rows, oracle-packed, run repeatedly): oracle "
                "NVFP4 activation quantisation + fp64 dequantise-then-dot")


class StackWorkload:
    """Every linear of a 64-layer dense decoder through nvq_decoder_stack."""

    kernel = "stack_pass"
    dtype = "nvfp4 x q8_0 (int32 subblock sums / exact fp16 operands, fp32 accumulate)"
    sources = ("nvq_stack.cpp", "gemv.cu", "gemm_tcgen05.cu", "quantize_q8_0.cu")
    unit = "tokens/s"

    def __init__(self, name, M):
        from bit_weight_quantized_nvq_b200 import workloads as wl
        self.name, self.M = name, M
        self.bound = "hbm" if M <= 16 else "tensor"
        self.metric = "nvfp4_q8_0_linear_stack_tokens_per_s"
        self.n_layers = wl.STACK_LAYERS
        self.linears = wl.STACK_LINEARS

    def setup(self, device):
        import torch
        from bit_weight_quantized_nvq_b200 import capi, workloads as wl
        self.capi = capi
        layer_host = []
        for name, W in wl.stack_layer_weights():
            codes, scales, g = capi.pack_nvfp4(W)
            layer_host.append((codes, scales, g))
            del W
        layers = []
        for _ in range(wl.STACK_LAYERS):
            layers.append([(torch.from_numpy(c).to(device), torch.from_numpy(s).to(device), g)
                           for c, s, g in layer_host])
        self.stack = capi.DecoderStack(layers, self.M, device=device)
        x = wl.stack_input(self.M)
        self.x = torch.from_numpy(x).to(device)
        self.x_host = torch.from_numpy(x).pin_memory()
        self.y_host = torch.empty(tuple(self.stack.outs[6].shape), dtype=torch.float32).pin_memory()

    def weight_bytes(self):
        return self.n_layers * sum(N * K * WEIGHT_BYTES_PER_ELEMENT for _, K, N in self.linears)

    def flops(self):
        return 2.0 * self.M * self.n_layers * sum(N * K for _, K, N in self.linears)

    def config(self):
        return {"workload": self.name, "M": self.M, "layers": self.n_layers,
                "linears_KN": {n: [K, N] for n, K, N in self.linears},
                "weights_GB": round(self.weight_bytes() / 1e9, 2),
                "dataflow": "per layer: Q8_0(x)->q,k,v; Q8_0(y_v)->o; Q8_0(y_o)->up,gate; "
                            "Q8_0(y_up)->down; every layer restarts from the same x",
                "l2": "inputs larger than L2 (17.9 GB of weights per pass)",
                "parallelism": "replicas"}

    def units_per_step(self):
        return float(self.M)                        # tokens

    def launches_per_step(self):
        if self.M == 1:
            # Q8_0 of the token, then the persistent stack kernel (64 layers a launch)
            return 1 + -(-self.n_layers // 64)
        if self.M <= 16:
            return (4 + 7) * self.n_layers
        # 4 quantisations and expansions, and the 7 GEMMs of every layer
        return self.n_layers * (8 + sum(gemm_launches(self.M, N, K) for _, K, N in self.linears))

    def step(self, stream, e2e=False):
        if e2e:
            self.x.copy_(self.x_host, non_blocking=True)
        self.stack.forward(self.x, stream=stream)
        if e2e:
            self.y_host.copy_(self.stack.outs[6], non_blocking=True)

    def e2e_bytes(self):
        return self.x.numel() * 4, self.stack.outs[6].numel() * 4

    def shape_timings(self, stream, reps):
        return None

    def oracle_tasks(self, rows):
        """One layer's 7 products on a row sample; units = tokens of the
        64-layer pass that this much work is worth (row fraction x layers)."""
        from bit_weight_quantized_nvq_b200 import workloads as wl
        toks = max(1, min(self.M, 4))
        total = sum(K * N for _, K, N in self.linears)
        tasks = []
        for i, (name, K, N) in enumerate(self.linears):
            def make(name=name, K=K, N=N, i=i):
                rng = np.random.default_rng(i)
                return (wl.weight_rows("stack", name, N, K, ORACLE_BASE_ROWS),
                        rng.standard_normal((toks, K)).astype(np.float32))
            base = oracle_base(("stack", self.name, K, N, name), make)
            tasks.append(sample_task(base, rows, toks * (K / total) / self.n_layers))
        return tasks

    def oracle_sample_desc(self, rows):
        toks = max(1, min(self.M, 4))
        return (f"{toks} token(s) x {rows} weight rows of each of the 7 linears of one layer "
                f"(the first {ORACLE_BASE_ROWS} rows, oracle-packed, run repeatedly; random "
                "activations), scaled to the 64-layer pass by the fraction of weights processed")


class W4A16Workload(GemvWorkload):
    """fp16-activation decode (W4A16): nvq_gemm_w4a16 over the decode-sweep
    shapes, one token; the activations are given in fp16 (no quantiser)."""

    kernel = "gemm_w4a16"
    sources = ("gemm_small.cu", "nvq_device.cuh", "tcgen05.cuh")   # the dominant kernel's code
    dtype = "nvfp4 x f16 (exact fp16 operands, fp32 accumulate)"
    metric = "nvfp4_f16_w4a16_weight_GBps"

    def setup(self, device):
        import torch
        super().setup(device)
        for c in self.cases:
            c["x"] = c["x"].half()
            c["x_host"] = c["x_host"].half().pin_memory()
            c["ws"] = torch.empty(
                int(self.capi.lib().nvq_gemm_w4a16_workspace_size(self.M, c["N"], c["K"])),
                dtype=torch.uint8, device=device)

    def config(self):
        cfg = super().config()
        cfg["activations"] = "fp16 N(0,1) (no quantisation)"
        cfg["path"] = "nvq_gemm_w4a16 (small-token tcgen05 schedule on fp16 activations)"
        return cfg

    def kernel_amount(self, K, N):
        return N * K * WEIGHT_BYTES_PER_ELEMENT + 2 * self.M * K + 4 * self.M * N

    def launches_per_step(self):
        return 3 * len(self.cases)       # fp16 operand layout, tcgen05 kernel, split-tile sum

    def dominant(self, c, codes, scales, stream):
        self.capi.gemm_w4a16(codes, scales, c["g"], c["x"], c["y"], c["ws"], stream=stream)

    def step(self, stream, e2e=False):
        for c in self.cases:
            if e2e:
                c["x"].copy_(c["x_host"], non_blocking=True)
            self.dominant(c, c["codes"], c["scales"], stream)
            if e2e:
                c["y_host"].copy_(c["y"], non_blocking=True)

    def e2e_bytes(self):
        return (sum(c["x"].numel() * 2 for c in self.cases),
                sum(c["y"].numel() * 4 for c in self.cases))

    def oracle_tasks(self, rows):
        tasks = []
        for K, N in self.shapes:
            def make(K=K, N=N):
                W, x = self.oracle_rows(K, N, ORACLE_BASE_ROWS)
                return W, x.astype(np.float16).view(np.uint16)
            base = oracle_base(("w4a16", self.name, K, N), make)
            tasks.append(sample_task(base, rows, K * WEIGHT_BYTES_PER_ELEMENT / 1e9))
        return tasks

    def oracle_sample_desc(self, rows):
        return (f"{rows} weight rows of each of the {len(self.shapes)} shapes (the first "
                f"{ORACLE_BASE_ROWS} rows, oracle-packed, run repeatedly), one fp16 token: "
                "oracle fp64 dequantise-then-dot")


class MoeWorkload:
    """Mixture-of-experts decode: Q8_0 of 16 tokens and nvq_moe_gemv."""

    kernel = "moe_gemv"
    dtype = "nvfp4 x q8_0 (int32 subblock sums, fp32 accumulate)"
    sources = ("gemv.cu", "nvq_device.cuh", "tcgen05.cuh")
    bound = "hbm"
    metric = "nvfp4_q8_0_moe_gemv_weight_GBps"
    unit = "GB/s"
    ROUTINGS = 8

    def __init__(self, name):
        from bit_weight_quantized_nvq_b200 import workloads as wl
        self.name = name
        self.E, self.N, self.K = wl.MOE_EXPERTS, wl.MOE_N, wl.MOE_K
        self.top_k, self.T = wl.MOE_TOP_K, wl.MOE_TOKENS

    def setup(self, device):
        import torch
        from bit_weight_quantized_nvq_b200 import capi, workloads as wl
        self.capi = capi
        E, N, K = self.E, self.N, self.K
        self.codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device=device)
        self.scales = torch.empty((E, N, K // 16), dtype=torch.uint8, device=device)
        g = np.empty(E, np.float32)
        for e in range(E):
            c, sc, g[e] = capi.pack_nvfp4(wl.moe_expert_weights(e))
            self.codes[e].copy_(torch.from_numpy(c))
            self.scales[e].copy_(torch.from_numpy(sc))
        self.g = torch.from_numpy(g).to(device)
        self.ids = [torch.from_numpy(wl.moe_routing(self.T, step=s)).to(device)
                    for s in range(self.ROUTINGS)]
        x = wl.moe_tokens(self.T)
        self.x = torch.from_numpy(x).to(device)
        self.x_host = torch.from_numpy(x).pin_memory()
        self.q = torch.empty((self.T, K), dtype=torch.int8, device=device)
        self.d = torch.empty((self.T, K // 32), dtype=torch.float16, device=device)
        self.y = torch.empty((self.T, self.top_k, N), dtype=torch.float32, device=device)
        self.y_host = torch.empty(tuple(self.y.shape), dtype=torch.float32).pin_memory()
        self.i = 0

    def config(self):
        return {"workload": self.name, "tokens": self.T, "experts": self.E,
                "top_k": self.top_k, "expert_KN": [self.K, self.N],
                "weights": "NVFP4 experts, N(0,0.02^2); routing uniform without replacement, "
                           f"{self.ROUTINGS} seeded routings used in turn",
                "activations": "fp32 N(0,1) -> Q8_0 on the GPU every step",
                "l2": "inputs larger than L2 (%.0f MB of expert rows per step, 453 MB of "
                      "experts)" % (self.weight_bytes() / 1e6),
                "parallelism": "replicas"}

    def weight_bytes(self):
        return self.T * self.top_k * self.N * self.K * WEIGHT_BYTES_PER_ELEMENT

    def units_per_step(self):
        return self.weight_bytes() / 1e9

    def kernel_amount(self):
        return (self.weight_bytes() + self.T * self.K * (1 + 2 / 32)
                + 4 * self.T * self.top_k * self.N + 4 * self.T * self.top_k)

    def launches_per_step(self):
        return 2

    def dominant(self, ids, stream):
        self.capi.moe_gemv(self.codes, self.scales, self.g, ids, self.q, self.d, self.y,
                           stream=stream)

    def step(self, stream, e2e=False):
        ids = self.ids[self.i % self.ROUTINGS]
        self.i += 1
        if e2e:
            self.x.copy_(self.x_host, non_blocking=True)
        self.capi.quantize_act_q8_0(self.x, self.q, self.d, stream=stream)
        self.dominant(ids, stream)
        if e2e:
            self.y_host.copy_(self.y, non_blocking=True)

    def e2e_bytes(self):
        return self.x.numel() * 4, self.y.numel() * 4

    def shape_timings(self, stream, reps):
        import torch
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            s = torch.cuda.current_stream()
            for i in range(reps):
                self.dominant(self.ids[i % self.ROUTINGS], s)
        graph.replay()
        ms = replay_ms(graph, stream)
        del graph
        return [{"K": self.K, "N": self.N * self.top_k * self.T, "us_per_launch": ms * 1e3 / reps,
                 "amount": self.kernel_amount(), "weight_copies": self.ROUTINGS}]

    def oracle_tasks(self, rows):
        from bit_weight_quantized_nvq_b200 import workloads as wl
        ids = wl.moe_routing(self.T, step=0)
        x = wl.moe_tokens(self.T)[:1]
        tasks = []
        for e in ids[0]:
            base = oracle_base(("moe", int(e)), lambda e=e: (
                wl.weight_rows("moe", f"expert{int(e)}", self.N, self.K, ORACLE_BASE_ROWS), x))
            tasks.append(sample_task(base, rows, self.K * WEIGHT_BYTES_PER_ELEMENT / 1e9))
        return tasks

    def oracle_sample_desc(self, rows):
        return (f"one token x {rows} weight rows of each of its {self.top_k} experts (the first "
                f"{ORACLE_BASE_ROWS} rows, oracle-packed, run repeatedly): oracle Q8_0 + fp64 "
                "dequantise-then-dot")


def make_workload(name: str):
    from bit_weight_quantized_nvq_b200 import workloads as wl
    if name == "decode_sweep":
        return GemvWorkload(name, wl.DECODE_SHAPES, 1, lambda K, N: wl.decode_case(K, N),
                            lambda K, N, r: (wl.weight_rows("decode_sweep", "W", N, K, r, True),
                                             wl.activations("decode_sweep", "x", 1, K)))
    if name == "gemv_4096":
        return GemvWorkload(name, [(4096, 4096)], 1, lambda K, N: wl.gemv_4096_case(),
                            lambda K, N, r: (wl.weight_rows("gemv_4096", "W", N, K, r),
                                             wl.activations("gemv_4096", "x", 1, K)))
    if name.startswith("small_batch_m"):
        M = int(name[len("small_batch_m"):])
        return SmallGemmWorkload(
            name, wl.SMALL_BATCH_SHAPES, M, lambda K, N: wl.small_batch_case(M, K, N),
            lambda K, N, r: (wl.weight_rows("small_batch", "W", N, K, r, True),
                             wl.activations("small_batch", "x", M, K, "student_t4")))
    if name.startswith("nvf4_prefill_m"):
        return Nvf4GemmWorkload(name, wl.PREFILL_SHAPES, int(name[len("nvf4_prefill_m"):]))
    if name.startswith("prefill_m"):
        return GemmWorkload(name, wl.PREFILL_SHAPES, int(name[len("prefill_m"):]))
    if name == "stack_decode":
        return StackWorkload(name, 1)
    if name == "stack_prefill":
        return StackWorkload(name, 2048)
    if name == "moe_decode":
        return MoeWorkload(name)
    if name == "w4a16_decode":
        return W4A16Workload(name, wl.DECODE_SHAPES, 1, lambda K, N: wl.decode_case(K, N),
                             lambda K, N, r: (wl.weight_rows("decode_sweep", "W", N, K, r, True),
                                              wl.activations("decode_sweep", "x", 1, K)))
    raise SystemExit(f"unknown workload {name!r}")


# ---------------------------------------------------------------------------
# measurement
# ---------------------------------------------------------------------------

def roofline_entry(wk, shapes, ms_per_step, peaks):
    """The dominant kernel's achieved rate against the measured peak."""
    if wk.bound == "hbm":
        scale, peak, unit, src = 1e9, peaks["hbm_gbs"], "GB/s", "hbm_gbs (copy)"
    elif getattr(wk, "peak_scale", None):
        scale, peak, unit, src = 1e12, peaks["bf16_tflops"] * wk.peak_scale, "TFLOP/s", \
            wk.peak_note
    else:
        scale, peak, unit, src = 1e12, peaks["bf16_tflops"], "TFLOP/s", \
            "bf16_tflops (burst; fp16 runs at the bf16 rate)"
    if shapes:
        amount = sum(s["amount"] for s in shapes)
        us = sum(s["us_per_launch"] for s in shapes)
        per_shape = [{"K": s["K"], "N": s["N"], "us": round(s["us_per_launch"], 3),
                      "achieved": round(s["amount"] / (s["us_per_launch"] / 1e6) / scale, 2),
                      "frac": round(s["amount"] / (s["us_per_launch"] / 1e6) / scale / peak, 4),
                      "weight_copies": s["weight_copies"]} for s in shapes]
        timing = ("each shape's dominant launch alone, back to back in an event-free CUDA "
                  "graph rotating through weight copies (>= 4x L2); sum of launch times "
                  f"{us:.2f} us per step vs the step's {ms_per_step * 1e3:.2f} us")
        launches = len(shapes)
        traffic = profiled_traffic(wk.kernel, wk.name, source_hash(*wk.sources))
    else:
        amount = wk.weight_bytes() if wk.bound == "hbm" else wk.flops()
        us = ms_per_step * 1e3
        per_shape = None
        timing = "one pass of the whole stack (the step) per unit"
        launches = 1
        traffic = None
    achieved = amount / (us / 1e6) / scale
    entry = {"bound": wk.bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
             "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": wk.kernel,
             "launches_per_step": launches, "avg_launch_us": round(us / launches, 3),
             "algorithmic_per_launch": amount / launches,
             "peak_source": f"{peaks['source']} MEASURED_PEAKS.json {src}",
             "step_achieved": round(amount / (ms_per_step / 1e3) / scale, 2),
             "step_frac": round(amount / (ms_per_step / 1e3) / scale / peak, 4),
             "timing": timing}
    if per_shape is not None:
        entry["per_shape"] = per_shape
    if wk.bound == "tensor" and wk.kernel == "gemm":
        entry["issued_frac"] = round(2 * achieved / peak, 4)   # hi and lo halves
    return entry


def measure(wk, args, dist: Dist, peaks, device, sampler):
    """Set up one workload, time its K steps, its dominant kernel per shape
    and its e2e path; returns the entry (times are maxima over ranks)."""
    import torch
    wk.setup(device)
    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        wk.step(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        s = torch.cuda.current_stream()
        for _ in range(args.steps):
            wk.step(s)
    graph.replay()                        # untimed replay (graph upload)
    torch.cuda.synchronize()
    dist.barrier()
    t_wall0 = time.time()
    ms = replay_ms(graph, stream)
    t_wall1 = time.time()
    dist.barrier()
    clocks = sampler.summary(t_wall0 - 0.05, t_wall1 + 0.05)
    del graph
    shapes = wk.shape_timings(stream, max(args.steps, 20))
    ms_max = dist.max(ms, device)
    ms_per_step = ms_max / args.steps
    if shapes:
        for s in shapes:
            s["us_per_launch"] = dist.max(s["us_per_launch"], device)
    roofline = roofline_entry(wk, shapes, ms_per_step, peaks)

    # e2e: the same K steps through the public API, eagerly, with copies
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
    e2e_ms = dist.max(e_start.elapsed_time(e_end), device)

    units = wk.units_per_step() * args.steps * dist.world
    h2d, d2h = wk.e2e_bytes()
    return {
        "metric": wk.metric, "value": round(units / (ms_max / 1e3), 3), "unit": wk.unit,
        "ms_per_step": round(ms_per_step, 5), "dtype": wk.dtype,
        "config": wk.config(),
        "e2e": {"value": round(units / (e2e_ms / 1e3), 3), "unit": wk.unit,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": "eager public API calls with pinned-host copies"},
        "gpu_launches": wk.launches_per_step() * args.steps,
        "roofline": roofline,
        "clocks": clocks,
    }


def cpu_baseline(wk, seconds: float, pool):
    """The oracle on a bounded sample of the workload: one host core, and
    every host core through the pool (when given)."""
    import threadpoolctl
    rows = 64
    with threadpoolctl.threadpool_limits(1):
        tasks = wk.oracle_tasks(rows)
        t0 = time.perf_counter()
        run_tasks_serial(tasks)
        t_small = time.perf_counter() - t0
        rows = int(max(64, rows * seconds / max(t_small, 1e-3)))
        tasks = wk.oracle_tasks(rows)
        t0 = time.perf_counter()
        units = run_tasks_serial(tasks)
        t = time.perf_counter() - t0
    entry = {"value": round(units / t, 6), "unit": wk.unit, "cores": 1, "kind": "oracle",
             "sample": wk.oracle_sample_desc(rows), "seconds": round(t, 2)}
    if pool is not None:
        rows_all = int(rows * max(1, pool.cores * 3 // 4))
        tasks = wk.oracle_tasks(rows_all)
        t0 = time.perf_counter()
        units = pool.run(tasks)
        t = time.perf_counter() - t0
        entry["all_cores"] = {"value": round(units / t, 6), "unit": wk.unit,
                              "cores": pool.cores, "kind": "oracle",
                              "sample": wk.oracle_sample_desc(rows_all),
                              "seconds": round(t, 2),
                              "how": "row blocks over a pool of spawned processes, one "
                                     "numpy thread each"}
    return entry


def run_nvq(args, dist: Dist):
    import gc

    import torch
    pool = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        pool = OraclePool()           # spawned before the first GPU call
    torch.cuda.set_device(dist.local_rank)
    device = torch.device("cuda", dist.local_rank)
    dist.init("nccl")
    peaks = load_peaks()
    # everything runs on one side stream (graphs are captured on it)
    stream = torch.cuda.Stream(device)
    torch.cuda.set_stream(stream)
    sampler = ClockSampler(dist.local_rank)
    sampler.start()
    time.sleep(0.3)

    names = [args.workload]
    if not args.no_sub:
        names += [n for n in SUB_WORKLOADS if n != args.workload]
    entries = {}
    for name in names:
        wk = make_workload(name)
        entry = measure(wk, args, dist, peaks, device, sampler)
        if pool is not None:
            entry["cpu_baseline"] = cpu_baseline(
                wk, args.cpu_seconds if name == args.workload else args.cpu_seconds / 4, pool)
        else:
            entry["cpu_baseline"] = None
        entries[name] = entry
        del wk
        gc.collect()
        torch.cuda.empty_cache()
    time.sleep(0.2)
    sampler.stop()
    if pool is not None:
        pool.close()

    main = entries.pop(args.workload)
    line = {
        "metric": main["metric"], "value": main["value"], "unit": main["unit"],
        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": main["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": main["dtype"],
        "data": "synthetic (seeded; shapes and distributions of the workload)",
        "config": main["config"],
        "impl": "nvq",
        "timing": ("CUDA graph of the K steps replayed once, events on the launching stream "
                   "before and after; no event nodes inside that replay"),
        "e2e": main["e2e"],
        "gpu_launches": main["gpu_launches"],
        "gpu_launches_all_workloads": main["gpu_launches"] + sum(e["gpu_launches"]
                                                                 for e in entries.values()),
        "roofline": main["roofline"],
        "cpu_baseline": main["cpu_baseline"],
        "clocks": main["clocks"],
    }
    if entries:
        line["workloads"] = entries
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


def run_reference(args, dist: Dist):
    """The oracle as the reference arm: rank 0 only, on the host cores."""
    if dist.rank != 0:
        return
    wk = make_workload(args.workload)
    pool = OraclePool()
    # size the per-step sample so that warm-up + timed steps take about
    # 6 * --cpu-seconds in total (a few minutes at most)
    budget = 6 * args.cpu_seconds / (args.steps + args.warmup)
    rows = 64
    tasks = wk.oracle_tasks(rows)
    t0 = time.perf_counter()
    pool.run(tasks)
    t_small = time.perf_counter() - t0
    rows = int(max(64, rows * budget / max(t_small, 1e-4)))
    tasks = wk.oracle_tasks(rows)
    for _ in range(args.warmup):
        pool.run(tasks)
    t0 = time.perf_counter()
    units = 0.0
    for _ in range(args.steps):
        units += pool.run(tasks)
    t = time.perf_counter() - t0
    pool.close()
    value = units / t
    desc = wk.oracle_sample_desc(rows)
    line = {
        "metric": wk.metric, "value": round(value, 6), "unit": wk.unit,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 (int64 subblock sums)",
        "data": "synthetic (seeded; a bounded sample of the workload per step)",
        "config": dict(wk.config(), sample_per_step=desc),
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 6), "unit": wk.unit, "cores": pool.cores,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 6), "unit": wk.unit,
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode_sweep")
    ap.add_argument("--impl", choices=["nvq", "reference"], default="nvq")
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
                    help="target duration of the headline's oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub", action="store_true",
                    help="measure only --workload (no other workloads in the line)")
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
