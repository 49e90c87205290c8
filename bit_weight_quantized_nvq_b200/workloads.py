"""Seeded synthetic inputs for the NVFP4 x Q8_0 kernels.

This module only draws random numbers: fp32 weight matrices and fp32
activations with the distributions of the workloads below.  It holds none of
the method's arithmetic (no quantisation, no packing, no dot products), so
both the library's tests and the independent CPU oracle can be fed from it.

Workloads (shapes are (K, N) of a weight W[N, K]; M is the token count):

* ``gemv_4096``     M=1, K=N=4096; W ~ N(0, 0.02^2), x ~ N(0, 1).
* ``decode_sweep``  M=1 over the linear shapes of a 27B-class dense decoder:
                    (5120, 5120), (5120, 25600), (25600, 5120), (5120, 152064);
                    W ~ N(0, 0.02^2) with 1 % of the input columns k scaled
                    x20 (stresses the UE4M3 scale range), x ~ N(0, 1).
* ``small_batch``   M in {2, 4, 8, 16} over (5120, 25600) and (25600, 5120);
                    weights as in ``decode_sweep``; x ~ Student-t(nu=4).
* ``prefill``       M in {256, 2048} over (5120, 5120), (5120, 25600) and
                    (25600, 5120); W ~ N(0, 0.02^2); x ~ N(0, 1) with 0.1 % of
                    the hidden channels scaled x50 in every token row.
* ``moe``           a mixture-of-experts layer at decode: 256 experts with
                    K = 2048 (hidden) and N = 1536 (the stacked gate and up
                    projections of a 768-wide expert), 6 experts per token,
                    16 tokens per step; W ~ N(0, 0.02^2) per expert, x ~
                    N(0, 1); each token's experts drawn uniformly without
                    replacement, seeded per step.
* ``stack``         the seven linears of one layer of a 64-layer dense
                    transformer (hidden 5120, gated MLP 25600): q, k, v, o
                    (5120, 5120), up and gate (5120, 25600), down (25600, 5120);
                    W ~ N(0, 0.02^2); layer input x ~ N(0, 1).

Seeding: every tensor has its own ``numpy.random.SeedSequence`` built from
the base seed 2026, a workload tag, a tensor tag and its shape.  Weights are
drawn in blocks of 1024 rows, each block from its own child sequence, so any
row block can be regenerated alone and large matrices are filled by several
threads.
"""
from __future__ import annotations

import math
import os
import zlib
from concurrent.futures import ThreadPoolExecutor

import numpy as np

BASE_SEED = 2026
ROW_BLOCK = 1024

DECODE_SHAPES = [(5120, 5120), (5120, 25600), (25600, 5120), (5120, 152064)]
SMALL_BATCH_MS = [2, 4, 8, 16]
SMALL_BATCH_SHAPES = [(5120, 25600), (25600, 5120)]
PREFILL_MS = [256, 2048]
PREFILL_SHAPES = [(5120, 5120), (5120, 25600), (25600, 5120)]
MOE_EXPERTS = 256
MOE_TOP_K = 6
MOE_K = 2048
MOE_N = 1536
MOE_TOKENS = 16
STACK_LAYERS = 64
STACK_HIDDEN = 5120
STACK_MLP = 25600
#: (name, K, N) of the seven linears of one layer, in execution order
STACK_LINEARS = [("q", 5120, 5120), ("k", 5120, 5120), ("v", 5120, 5120),
                 ("o", 5120, 5120), ("up", 5120, 25600),
                 ("gate", 5120, 25600), ("down", 25600, 5120)]

WEIGHT_STD = 0.02
COLUMN_BOOST_FRACTION = 0.01
COLUMN_BOOST = 20.0
OUTLIER_FRACTION = 0.001
OUTLIER_BOOST = 50.0


def _tag(s: str) -> int:
    return zlib.crc32(s.encode("utf-8"))


def seed_sequence(workload: str, tensor: str, *shape: int) -> np.random.SeedSequence:
    """The seed sequence of one tensor of one workload."""
    return np.random.SeedSequence([BASE_SEED, _tag(workload), _tag(tensor),
                                   *[int(v) for v in shape]])


def boosted_columns(workload: str, tensor: str, K: int) -> np.ndarray:
    """Sorted distinct input-column indices (ceil(1 % of K)) scaled x20."""
    rng = np.random.Generator(np.random.PCG64(
        seed_sequence(workload, tensor + "/columns", K)))
    n = math.ceil(COLUMN_BOOST_FRACTION * K)
    return np.sort(rng.choice(K, size=n, replace=False))


def outlier_channels(workload: str, tensor: str, K: int) -> np.ndarray:
    """Sorted distinct hidden-channel indices (ceil(0.1 % of K)) scaled x50."""
    rng = np.random.Generator(np.random.PCG64(
        seed_sequence(workload, tensor + "/outliers", K)))
    n = math.ceil(OUTLIER_FRACTION * K)
    return np.sort(rng.choice(K, size=n, replace=False))


def _fill_rows(ss: np.random.SeedSequence, out: np.ndarray, b: int,
               std: float) -> None:
    rng = np.random.Generator(np.random.PCG64(ss.spawn(b + 1)[b]))
    rows = out[b * ROW_BLOCK:(b + 1) * ROW_BLOCK]
    rng.standard_normal(out=rows, dtype=np.float32)
    rows *= np.float32(std)


def weights(workload: str, tensor: str, N: int, K: int,
            boost_columns: bool = False, threads: int | None = None) -> np.ndarray:
    """fp32 W[N, K] ~ N(0, 0.02^2); optionally 1 % of the columns x20."""
    ss = seed_sequence(workload, tensor, N, K)
    out = np.empty((N, K), dtype=np.float32)
    nblocks = (N + ROW_BLOCK - 1) // ROW_BLOCK
    threads = threads or min(16, os.cpu_count() or 1)
    if nblocks == 1 or threads == 1:
        for b in range(nblocks):
            _fill_rows(ss, out, b, WEIGHT_STD)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda b: _fill_rows(ss, out, b, WEIGHT_STD),
                        range(nblocks)))
    if boost_columns:
        out[:, boosted_columns(workload, tensor, K)] *= np.float32(COLUMN_BOOST)
    return out


def weight_rows(workload: str, tensor: str, N: int, K: int, rows: int,
                boost_columns: bool = False) -> np.ndarray:
    """The first `rows` rows of weights(workload, tensor, N, K, ...), drawn
    without generating the rest of the matrix (row blocks have their own
    seed sequences)."""
    rows = min(rows, N)
    ss = seed_sequence(workload, tensor, N, K)
    nblocks = (rows + ROW_BLOCK - 1) // ROW_BLOCK
    out = np.empty((nblocks * ROW_BLOCK, K), dtype=np.float32)
    for b in range(nblocks):
        _fill_rows(ss, out, b, WEIGHT_STD)
    out = out[:rows]
    if boost_columns:
        out[:, boosted_columns(workload, tensor, K)] *= np.float32(COLUMN_BOOST)
    return out


def activations(workload: str, tensor: str, M: int, K: int,
                dist: str = "normal", outliers: bool = False) -> np.ndarray:
    """fp32 x[M, K]: N(0, 1) or Student-t(nu=4); optionally 0.1 % of the
    channels x50 in every row."""
    rng = np.random.Generator(np.random.PCG64(seed_sequence(workload, tensor, M, K)))
    if dist == "normal":
        x = rng.standard_normal((M, K), dtype=np.float32)
    elif dist == "student_t4":
        x = rng.standard_t(4.0, size=(M, K)).astype(np.float32)
    else:
        raise ValueError(f"unknown activation distribution {dist!r}")
    if outliers:
        x[:, outlier_channels(workload, tensor, K)] *= np.float32(OUTLIER_BOOST)
    return x


def decode_case(K: int, N: int, M: int = 1, workload: str = "decode_sweep"):
    """(W, x) of one decode-sweep shape (boosted columns, N(0,1) x)."""
    W = weights(workload, "W", N, K, boost_columns=True)
    x = activations(workload, "x", M, K, "normal")
    return W, x


def gemv_4096_case():
    """(W, x) of the single K=N=4096, M=1 GEMV."""
    return (weights("gemv_4096", "W", 4096, 4096),
            activations("gemv_4096", "x", 1, 4096, "normal"))


def small_batch_case(M: int, K: int, N: int):
    """(W, x) of one small-batch shape (boosted columns, Student-t x)."""
    return (weights("small_batch", "W", N, K, boost_columns=True),
            activations("small_batch", "x", M, K, "student_t4"))


def prefill_case(M: int, K: int, N: int):
    """(W, x) of one prefill shape (plain W, N(0,1) x with outliers)."""
    return (weights("prefill", "W", N, K),
            activations("prefill", "x", M, K, "normal", outliers=True))


def stack_layer_weights():
    """fp32 weights of the seven linears of one layer, in execution order."""
    return [(name, weights("stack", name, N, K)) for name, K, N in STACK_LINEARS]


def stack_input(M: int):
    """fp32 layer input x[M, 5120] ~ N(0, 1)."""
    return activations("stack", "x", M, STACK_HIDDEN, "normal")


def moe_expert_weights(e: int, N: int = MOE_N, K: int = MOE_K, workload: str = "moe") -> np.ndarray:
    """fp32 W_e[N, K] of expert e ~ N(0, 0.02^2)."""
    return weights(workload, f"expert{e}", N, K)


def moe_routing(T: int, top_k: int = MOE_TOP_K, E: int = MOE_EXPERTS, step: int = 0,
                workload: str = "moe") -> np.ndarray:
    """int32 ids[T, top_k]: each token's experts, distinct, uniform."""
    rng = np.random.Generator(np.random.PCG64(seed_sequence(workload, "routing", T, top_k, E, step)))
    return np.stack([rng.choice(E, size=top_k, replace=False) for _ in range(T)]).astype(np.int32)


def moe_tokens(T: int = MOE_TOKENS, K: int = MOE_K, workload: str = "moe") -> np.ndarray:
    """fp32 x[T, K] ~ N(0, 1)."""
    return activations(workload, "x", T, K, "normal")
