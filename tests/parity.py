"""Helpers shared by the GPU parity tests: run the CUDA path and the oracle
on the same seeded inputs and compare.

The CUDA path packs weights with the library's host packer and quantises
activations with its GPU quantiser; the oracle packs and quantises with its
own code.  Both sides start from the same fp32 inputs drawn by
``bit_weight_quantized_nvq_b200.workloads``; the packed bytes and the Q8_0
codes are compared bit for bit before any output is compared.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as o
from bit_weight_quantized_nvq_b200 import capi


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def sample_rows(N: int, n: int, seed: int) -> np.ndarray:
    """First, last and n random rows (sorted, distinct)."""
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(N, size=min(n, N), replace=False).tolist())
    rows.update({0, N - 1})
    return np.array(sorted(rows))


class Packed:
    """A weight matrix packed by the library (device copy) with the oracle's
    packing of selected rows next to it."""

    def __init__(self, W: np.ndarray, rows: np.ndarray | None = None):
        codes, scales, g = capi.pack_nvfp4(W)
        self.N, self.K = W.shape
        self.g = g
        self.codes = to_dev(codes)
        self.scales = to_dev(scales)
        self.rows = np.arange(self.N) if rows is None else rows
        g_ref = o.nvfp4_tensor_scale(W)
        self.ref_codes, self.ref_scales, self.ref_g = o.pack_nvfp4(W[self.rows], g=g_ref)
        assert np.float32(g) == self.ref_g
        assert np.array_equal(codes[self.rows], self.ref_codes)
        assert np.array_equal(scales[self.rows], self.ref_scales)


def quantize_both(x: np.ndarray):
    """GPU and oracle Q8_0 of x; asserts they are bit-identical."""
    xd = to_dev(x)
    q, d = capi.quantize_act_q8_0(xd)
    torch.cuda.synchronize()
    q_ref, d_ref = o.quantize_q8_0(x)
    q_h = q.cpu().numpy()
    d_h = d.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(q_h, q_ref), "Q8_0 codes differ"
    assert np.array_equal(d_h, d_ref), "Q8_0 scales differ"
    return q, d, q_ref, d_ref


def reference(P: Packed, q_ref, d_ref):
    """Oracle y (fp64), sum|terms| and integer sums on P's selected rows."""
    y = o.dot_fp64(P.ref_codes, P.ref_scales, P.ref_g, q_ref, d_ref)
    isum = o.subblock_sums(P.ref_codes, q_ref)
    sa = o.sum_abs_terms(isum, P.ref_scales, P.ref_g, d_ref)
    return y, sa, isum


def assert_within_tolerance(y_gpu: np.ndarray, y_ref: np.ndarray, sa: np.ndarray):
    """|y_gpu - y_ref| <= 1e-5 * sum|terms| + 1e-6 per element, plus the
    false-pass guard: the reference is not identically zero."""
    assert y_gpu.shape == y_ref.shape
    assert np.all(np.isfinite(y_gpu))
    assert np.any(sa > 0) and np.any(y_ref != 0), "degenerate reference"
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    tol = o.tolerance(sa)
    bad = err > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{bad.sum()} of {bad.size} outside tolerance; first at {tuple(i)}: "
            f"gpu={y_gpu[tuple(i)]!r} ref={y_ref[tuple(i)]!r} tol={tol[tuple(i)]!r}")
    return float((err / np.maximum(tol, 1e-300)).max())
