#!/usr/bin/env python
"""Benchmark of the NVFP4 x Q8_0 kernels on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl nvq|reference]

Prints ONE JSON line on rank 0.

Workloads (``--workload``):
  decode_sweep (default)  one step quantises one token's activations (Q8_0)
                          and runs the decode GEMV for each of the four
                          linear shapes of a 27B-class dense decoder,
                          (K, N) = (5120, 5120), (5120, 25600), (25600, 5120),
                          (5120, 152064).  Metric: weight GB/s (NVFP4 weight
                          bytes N*K*0.5625 streamed per second).
  gemv_4096               M=1, K=N=4096.
  small_batch_m{2,4,8,16} decode GEMV at M tokens, (5120, 25600), (25600, 5120).
  prefill_m{256,2048}     Q8_0 + tcgen05 GEMM over (5120, 5120), (5120, 25600),
                          (25600, 5120).  Metric: algorithmic TFLOP/s 2*M*N*K.
  stack_decode            all 448 linears of a 64-layer dense decoder (17.9 GB
                          of NVFP4 weights resident), one token.  Metric:
                          tokens/s of the linear layers.
  stack_prefill           the same stack for 2048 tokens.

Timing: W untimed eager warm-up steps; the K timed steps are captured once
into a CUDA graph (the public entry points are graph-capturable: they only
enqueue work) and replayed inside the timed region, bracketed by a barrier
and a device synchronize and timed with CUDA events on the launching stream;
the time is the max over ranks.  The dominant kernel of every step is
bracketed by its own (graph-recorded) events for the roofline entry.  One
step's weights exceed the 126 MB L2 in every workload (600 MB for the decode
sweep), so no L2 flush is inserted.  ``e2e`` runs the same K steps through
the public Python API eagerly, with each step's activations copied from
pinned host memory and its outputs copied back inside the timed region (the
weights are resident model parameters).

Multi-GPU (``torchrun --nproc-per-node N``): every rank runs the same
workload on its own GPU with no data exchange (independent replicas; the
only collectives are the timing barrier and max).  ``value`` is the units of
all ranks divided by the max time; ``scaling`` is "weak".

``--impl reference`` times the plain CPU oracle on the host (rank 0 only),
each step a bounded sample of the same workload, on the same metric.
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
            inside, window = self.samples, "whole run (timed region shorter than one sample)"
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


class EventLog:
    """Start/stop events around the dominant kernel of each step; created
    external so that they become timestamp nodes when captured in a graph."""

    def __init__(self):
        self.pairs = []
        self._open = None

    def begin(self, stream):
        import torch
        ev = torch.cuda.Event(enable_timing=True, external=True)
        ev.record(stream)
        self._open = ev

    def end(self, stream, amount):
        import torch
        ev = torch.cuda.Event(enable_timing=True, external=True)
        ev.record(stream)
        self.pairs.append((self._open, ev, amount))
        self._open = None

    def totals(self):
        ms = sum(a.elapsed_time(b) for a, b, _ in self.pairs)
        amount = sum(x for _, _, x in self.pairs)
        return ms, amount, len(self.pairs)


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

class GemvWorkload:
    """M-token decode GEMVs over a list of (K, N) shapes; one step quantises
    each shape's activations and runs its GEMV."""

    kernel = "gemv"
    sources = ("gemv.cu", "nvq_device.cuh", "tcgen05.cuh")
    bound = "hbm"
    metric = "nvfp4_q8_0_gemv_weight_GBps"
    unit = "GB/s"

    def __init__(self, name, shapes, M, make_case):
        self.name, self.shapes, self.M, self.make_case = name, shapes, M, make_case

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
        act = "fp32 -> Q8_0 on the GPU every step (nvq_quantize_act_q8_0)"
        return {"workload": self.name, "M": self.M,
                "shapes_KN": [list(s) for s in self.shapes],
                "weights": "NVFP4 (E2M1 + UE4M3 per 16 + fp32 g), N(0,0.02^2)",
                "activations": act,
                "l2": "inputs larger than L2 (weights of one step %.0f MB > 126 MB)"
                      % (self.weight_bytes() / 1e6),
                "parallelism": "replicas"}

    def weight_bytes(self):
        return sum(N * K * WEIGHT_BYTES_PER_ELEMENT for K, N in self.shapes)

    def units_per_step(self):
        return self.weight_bytes() / 1e9          # GB

    def kernel_amount(self, c):
        """Algorithmic bytes of one GEMV launch: NVFP4 weights, the
        activations (fp32 when quantised inside the kernel, else Q8_0) and
        the fp32 output."""
        M, K, N = self.M, c["K"], c["N"]
        return N * K * WEIGHT_BYTES_PER_ELEMENT + M * K * (1 + 2 / 32) + 4 * M * N

    def launches_per_step(self):
        return 2 * len(self.cases)

    def step(self, stream, log=None, e2e=False):
        capi = self.capi
        for c in self.cases:
            if e2e:
                c["x"].copy_(c["x_host"], non_blocking=True)
            capi.quantize_act_q8_0(c["x"], c["q"], c["d"], stream=stream)
            if log is not None:
                log.begin(stream)
            capi.gemv(c["codes"], c["scales"], c["g"], c["q"], c["d"], c["y"], stream=stream)
            if log is not None:
                log.end(stream, self.kernel_amount(c))
            if e2e:
                c["y_host"].copy_(c["y"], non_blocking=True)

    def e2e_bytes(self):
        return (sum(c["x"].numel() * 4 for c in self.cases),
                sum(c["y"].numel() * 4 for c in self.cases))

    # --- CPU oracle sample ---------------------------------------------------
    def oracle_prepare(self, size):
        import oracle as o
        self.o = o
        self.samples = []
        for K, N in self.shapes:
            W, x = self.make_case(K, N)
            g = o.nvfp4_tensor_scale(W)
            r = min(size, N)
            codes, scales, _ = o.pack_nvfp4(W[:r], g=g)
            del W
            self.samples.append((K, r, codes, scales, g, x))

    def oracle_step(self):
        o = self.o
        gb = 0.0
        for K, r, codes, scales, g, x in self.samples:
            q, d = o.quantize_q8_0(x)
            o.dot_fp64(codes, scales, g, q, d)
            gb += r * K * WEIGHT_BYTES_PER_ELEMENT / 1e9
        return gb

    def oracle_sample_desc(self, size):
        return (f"first {size} rows of each of the {len(self.shapes)} shapes, M={self.M}: "
                "oracle Q8_0 quantisation + fp64 dequantise-then-dot")


class GemmWorkload:
    """Prefill: Q8_0 of M tokens and the tcgen05 GEMM for each shape."""

    kernel = "gemm"
    sources = ("gemm_tcgen05.cu", "nvq_device.cuh", "tcgen05.cuh")
    bound = "tensor"
    metric = "nvfp4_q8_0_prefill_gemm_TFLOPs"
    unit = "TFLOP/s"

    def __init__(self, name, shapes, M):
        self.name, self.shapes, self.M = name, shapes, M

    def setup(self, device):
        import torch
        from bit_weight_quantized_nvq_b200 import capi, workloads as wl
        self.capi = capi
        self.cases = []
        M = self.M
        for K, N in self.shapes:
            W, x = wl.prefill_case(M, K, N)
            codes, scales, g = capi.pack_nvfp4(W)
            del W
            c = {"K": K, "N": N, "g": g,
                 "codes": torch.from_numpy(codes).to(device),
                 "scales": torch.from_numpy(scales).to(device),
                 "x": torch.from_numpy(x).to(device),
                 "x_host": torch.from_numpy(x).pin_memory(),
                 "q": torch.empty((M, K), dtype=torch.int8, device=device),
                 "d": torch.empty((M, K // 32), dtype=torch.float16, device=device),
                 "y": torch.empty((M, N), dtype=torch.float32, device=device),
                 "ws": torch.empty(capi.gemm_workspace_size(M, N, K), dtype=torch.uint8,
                                   device=device)}
            c["y_host"] = torch.empty((M, N), dtype=torch.float32).pin_memory()
            self.cases.append(c)

    def config(self):
        return {"workload": self.name, "M": self.M,
                "shapes_KN": [list(s) for s in self.shapes],
                "weights": "NVFP4, N(0,0.02^2)",
                "activations": "fp32 N(0,1), 0.1% channels x50 -> Q8_0 on the GPU every step",
                "l2": "inputs larger than L2 (activations and weights of one step > 126 MB)",
                "parallelism": "replicas"}

    def flops(self, c):
        return 2.0 * self.M * c["N"] * c["K"]

    def units_per_step(self):
        return sum(2.0 * self.M * N * K for K, N in self.shapes) / 1e12   # TFLOP

    def kernel_amount(self, c):
        return self.flops(c)

    def launches_per_step(self):
        return 3 * len(self.cases)       # quantise, expand, tcgen05 GEMM

    def step(self, stream, log=None, e2e=False):
        capi = self.capi
        for c in self.cases:
            if e2e:
                c["x"].copy_(c["x_host"], non_blocking=True)
            capi.quantize_act_q8_0(c["x"], c["q"], c["d"], stream=stream)
            if log is not None:
                log.begin(stream)
            capi.gemm(c["codes"], c["scales"], c["g"], c["q"], c["d"], c["y"], c["ws"],
                      stream=stream)
            if log is not None:
                log.end(stream, self.kernel_amount(c))
            if e2e:
                c["y_host"].copy_(c["y"], non_blocking=True)

    def e2e_bytes(self):
        return (sum(c["x"].numel() * 4 for c in self.cases),
                sum(c["y"].numel() * 4 for c in self.cases))

    def oracle_prepare(self, size):
        import oracle as o
        from bit_weight_quantized_nvq_b200 import workloads as wl
        self.o = o
        self.samples = []
        toks = max(1, min(self.M, size // 64))
        for K, N in self.shapes:
            W, x = wl.prefill_case(self.M, K, N)
            g = o.nvfp4_tensor_scale(W)
            r = min(size, N)
            codes, scales, _ = o.pack_nvfp4(W[:r], g=g)
            del W
            self.samples.append((K, r, codes, scales, g, x[:toks]))

    def oracle_step(self):
        o = self.o
        tf = 0.0
        for K, r, codes, scales, g, x in self.samples:
            q, d = o.quantize_q8_0(x)
            o.dot_fp64(codes, scales, g, q, d)
            tf += 2.0 * x.shape[0] * r * K / 1e12
        return tf

    def oracle_sample_desc(self, size):
        toks = max(1, min(self.M, size // 64))
        return (f"{toks} tokens x first {size} rows of each of the {len(self.shapes)} shapes: "
                "oracle Q8_0 + fp64 dequantise-then-dot")


class StackWorkload:
    """Every linear of a 64-layer dense decoder through nvq_decoder_stack."""

    kernel = "stack_pass"
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
        self.layer_host = []
        for name, W in wl.stack_layer_weights():
            codes, scales, g = capi.pack_nvfp4(W)
            self.layer_host.append((codes, scales, g))
            del W
        layers = []
        for _ in range(wl.STACK_LAYERS):
            layers.append([(torch.from_numpy(c).to(device), torch.from_numpy(s).to(device), g)
                           for c, s, g in self.layer_host])
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

    def kernel_amount(self, _=None):
        return self.weight_bytes() if self.bound == "hbm" else self.flops()

    def launches_per_step(self):
        per_layer = 4 + 7 + (4 if self.M > 16 else 0)
        return per_layer * self.n_layers

    def step(self, stream, log=None, e2e=False):
        if e2e:
            self.x.copy_(self.x_host, non_blocking=True)
        if log is not None:
            log.begin(stream)
        self.stack.forward(self.x, stream=stream)
        if log is not None:
            log.end(stream, self.kernel_amount())
        if e2e:
            self.y_host.copy_(self.stack.outs[6], non_blocking=True)

    def e2e_bytes(self):
        return self.x.numel() * 4, self.stack.outs[6].numel() * 4

    def oracle_prepare(self, size):
        import oracle as o
        from bit_weight_quantized_nvq_b200 import workloads as wl
        self.o = o
        self.samples = []
        toks = max(1, min(self.M, size // 256))
        for name, W in wl.stack_layer_weights():
            g = o.nvfp4_tensor_scale(W)
            r = min(size, W.shape[0])
            codes, scales, _ = o.pack_nvfp4(W[:r], g=g)
            self.samples.append((W.shape[1], W.shape[0], r, codes, scales, g))
        self.x_s = wl.stack_input(self.M)[:toks]

    def oracle_step(self):
        """One layer's 7 products on a row sample; returns tokens of the
        64-layer pass that this much work is worth (row fraction x layers)."""
        o = self.o
        frac = 0.0
        rng = np.random.default_rng(0)
        for K, N, r, codes, scales, g in self.samples:
            x = rng.standard_normal((self.x_s.shape[0], K)).astype(np.float32)
            q, d = o.quantize_q8_0(x)
            o.dot_fp64(codes, scales, g, q, d)
            frac += r * K / sum(KK * NN for _, KK, NN in self.linears)
        return self.x_s.shape[0] * frac / self.n_layers

    def oracle_sample_desc(self, size):
        toks = max(1, min(self.M, size // 256))
        return (f"{toks} token(s) x first {size} rows of each of the 7 linears of one layer "
                "(random activations), scaled to the 64-layer pass by the fraction of weights "
                "processed")


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
    if name.startswith("prefill_m"):
        return GemmWorkload(name, wl.PREFILL_SHAPES, int(name[len("prefill_m"):]))
    if name == "stack_decode":
        return StackWorkload(name, 1)
    if name == "stack_prefill":
        return StackWorkload(name, 2048)
    raise SystemExit(f"unknown workload {name!r}")


# ---------------------------------------------------------------------------
# timing
# ---------------------------------------------------------------------------

def capture_steps(wk, steps: int, stream, events: bool):
    """A CUDA graph of `steps` steps, optionally with an event pair around
    the dominant kernel of every step."""
    import torch
    log = EventLog() if events else None
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        s = torch.cuda.current_stream()
        for _ in range(steps):
            wk.step(s, log)
    return graph, log


def roofline_entry(wk, log, peaks):
    """The dominant kernel's achieved rate.  Its launch durations come from a
    replay whose graph has an event pair around every such launch; an event
    record node adds a little latency to the launch it brackets, so this is
    a conservative figure.  `step_achieved` divides the same algorithmic
    amount by the event-free step time instead (it also charges the other
    kernels of the step to the dominant one: a lower bound too)."""
    kernel_ms, amount, n = log.totals()
    src_hash = source_hash(*wk.sources)
    traffic = profiled_traffic(wk.kernel, wk.name, src_hash)
    if wk.bound == "hbm":
        achieved = amount / (kernel_ms / 1e3) / 1e9
        peak, unit, src = peaks["hbm_gbs"], "GB/s", "hbm_gbs (copy)"
    else:
        achieved = amount / (kernel_ms / 1e3) / 1e12
        peak, unit, src = peaks["bf16_tflops"], "TFLOP/s", "bf16_tflops (burst; fp16 runs at the bf16 rate)"
    entry = {"bound": wk.bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
             "frac": round(achieved / peak, 4), "traffic": traffic,
             "kernel": wk.kernel, "launches": n,
             "avg_launch_us": round(kernel_ms * 1e3 / max(1, n), 3),
             "algorithmic_per_launch": amount / max(1, n),
             "peak_source": f"{peaks['source']} MEASURED_PEAKS.json {src}"}
    if wk.bound == "tensor" and wk.kernel == "gemm":
        entry["issued_frac"] = round(2 * achieved / peak, 4)   # hi and lo halves
    entry["timing"] = ("launch durations from a second replay of the same steps with an "
                       "event pair around every dominant-kernel launch")
    return entry


def run_nvq(args, dist: Dist):
    import torch
    torch.cuda.set_device(dist.local_rank)
    device = torch.device("cuda", dist.local_rank)
    dist.init("nccl")
    peaks = load_peaks()
    wk = make_workload(args.workload)
    wk.setup(device)
    # graphs are captured on a side stream; everything runs on it
    stream = torch.cuda.Stream(device)
    torch.cuda.set_stream(stream)

    for _ in range(args.warmup):
        wk.step(stream)
    torch.cuda.synchronize()
    graph, _ = capture_steps(wk, args.steps, stream, events=False)
    graph_ev, log = capture_steps(wk, args.steps, stream, events=True)
    graph.replay()                        # untimed replays (graph upload)
    graph_ev.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(dist.local_rank)
    sampler.start()
    time.sleep(0.35)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start.record(stream)
    graph.replay()
    end.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    dist.barrier()
    ms = start.elapsed_time(end)
    graph_ev.replay()                     # the dominant kernel's launch durations
    torch.cuda.synchronize()
    t_wall2 = time.time()
    roofline = roofline_entry(wk, log, peaks)
    roofline["step_achieved"] = round(
        log.totals()[1] / (ms / 1e3) / (1e9 if wk.bound == "hbm" else 1e12), 2)
    time.sleep(0.25)
    sampler.stop()
    clocks = sampler.summary(t_wall0 - 0.1, t_wall2 + 0.1)
    del graph, graph_ev

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
    e2e_ms = e_start.elapsed_time(e_end)

    ms_max = dist.max(ms, device)
    e2e_ms_max = dist.max(e2e_ms, device)
    units = wk.units_per_step() * args.steps * dist.world
    value = units / (ms_max / 1e3)
    e2e_value = units / (e2e_ms_max / 1e3)

    extra = {}
    if args.workload == "decode_sweep" and dist.world == 1 and not args.no_prefill_summary:
        extra["prefill_gemm"] = prefill_summary(device, peaks)

    cpu = None   # the oracle's host-core baseline: rank 0 of a 1-GPU run only
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wk, args.cpu_seconds)

    h2d, d2h = wk.e2e_bytes()
    line = {
        "metric": wk.metric, "value": round(value, 3), "unit": wk.unit,
        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 x q8_0 (int32 subblock sums / exact fp16 operands, fp32 accumulate)",
        "data": "synthetic (seeded; shapes and distributions of the workload)",
        "config": wk.config(),
        "impl": "nvq",
        "timing": ("CUDA graph of the K steps replayed once, events on the launching stream "
                   "before and after; no event nodes inside that replay"),
        "e2e": {"value": round(e2e_value, 3), "unit": wk.unit,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": "eager public API calls with pinned-host copies"},
        "gpu_launches": wk.launches_per_step() * args.steps,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "clocks": clocks,
    }
    line.update(extra)
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


def prefill_summary(device, peaks):
    """The prefill GEMM at 2048 tokens, timed the same way (graph replay),
    reported next to the decode line."""
    import torch
    wk = make_workload("prefill_m2048")
    wk.setup(device)
    stream = torch.cuda.current_stream(device)   # the side stream set by run_nvq
    for _ in range(3):
        wk.step(stream)
    torch.cuda.synchronize()
    steps = 10
    graph, _ = capture_steps(wk, steps, stream, events=False)
    graph_ev, log = capture_steps(wk, steps, stream, events=True)
    graph.replay()
    graph_ev.replay()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    graph.replay()
    end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    graph_ev.replay()
    torch.cuda.synchronize()
    roof = roofline_entry(wk, log, peaks)
    roof["step_achieved"] = round(log.totals()[1] / (ms / 1e3) / 1e12, 2)
    out = {"workload": "prefill_m2048", "shapes_KN": [list(s) for s in wk.shapes],
           "step_TFLOPs": round(wk.units_per_step() * steps / (ms / 1e3), 2),
           "roofline": roof}
    del graph, graph_ev, wk
    torch.cuda.empty_cache()
    return out


def cpu_baseline(wk, seconds: float):
    """The oracle, timed on one host core on a bounded sample of the workload."""
    import threadpoolctl
    size = 64
    with threadpoolctl.threadpool_limits(1):
        wk.oracle_prepare(size)
        t0 = time.perf_counter()
        wk.oracle_step()
        t_small = time.perf_counter() - t0
        size = int(max(64, min(65536, size * seconds / max(t_small, 1e-3))))
        wk.oracle_prepare(size)
        t0 = time.perf_counter()
        units = wk.oracle_step()
        t = time.perf_counter() - t0
    return {"value": round(units / t, 6), "unit": wk.unit, "cores": 1, "kind": "oracle",
            "sample": wk.oracle_sample_desc(size), "seconds": round(t, 2)}


def run_reference(args, dist: Dist):
    """The oracle as the reference arm: rank 0 only, on the host cores."""
    if dist.rank != 0:
        return
    import threadpoolctl
    wk = make_workload(args.workload)
    # size the per-step sample so that warm-up + timed steps take about
    # 6 * --cpu-seconds in total (a few minutes at most)
    budget = 6 * args.cpu_seconds / (args.steps + args.warmup)
    size = 64
    with threadpoolctl.threadpool_limits(1):
        wk.oracle_prepare(size)
        t0 = time.perf_counter()
        wk.oracle_step()
        t_small = time.perf_counter() - t0
        size = int(max(8, min(65536, size * budget / max(t_small, 1e-4))))
        wk.oracle_prepare(size)
        for _ in range(args.warmup):
            wk.oracle_step()
        t0 = time.perf_counter()
        units = 0.0
        for _ in range(args.steps):
            units += wk.oracle_step()
        t = time.perf_counter() - t0
    value = units / t
    desc = wk.oracle_sample_desc(size)
    line = {
        "metric": wk.metric, "value": round(value, 6), "unit": wk.unit,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 (int64 subblock sums)",
        "data": "synthetic (seeded; a bounded sample of the workload per step)",
        "config": dict(wk.config(), sample_per_step=desc),
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 6), "unit": wk.unit, "cores": 1,
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
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="decode_sweep")
    ap.add_argument("--impl", choices=["nvq", "reference"], default="nvq")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target duration of the oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill-summary", action="store_true")
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
