"""Helpers shared by the GPU parity tests: run the CUDA path and the oracle
on the same seeded inputs and compare.

The CUDA path packs weights with the library's host packer and quantises
activations with its GPU quantiser; the oracle packs and quantises with its
own code.  Both sides start from the same fp32 inputs drawn by
``bit_weight_quantized_nvq_b200.workloads``; the packed bytes and the Q8_0
codes are compared bit for bit before any output is compared.
"""
from __future__ import annotations

import os

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


#: (test id, max err/tol) of every tolerance comparison in this session,
#: summarised at the end of the run (tests/conftest.py)
MARGINS: list[tuple[str, float]] = []


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
    ratio = float((err / np.maximum(tol, 1e-300)).max())
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    MARGINS.append((test, ratio))
    return ratio


# ---------------------------------------------------------------------------
# chained products (the decoder stack): tolerance propagation
# ---------------------------------------------------------------------------

def requant_bound(x_ref: np.ndarray, x_tol: np.ndarray) -> np.ndarray:
    """Bound on |a_gpu - a_ref| for a = fp16(d)*q when the quantiser's input
    is known only to within x_tol of the oracle's x_ref (fp32 values).

    Per 32-block, the largest |x| lies within the tolerance of the oracle's,
    so d32 and the fp16 d lie in an interval; every element's x/d32 lies in
    an interval, and rint is monotone, so q lies in [q_lo, q_hi].  The bound
    is the largest distance of d*q over those intervals from the oracle's
    d_ref*q_ref.  It is zero wherever neither d nor q can change (the usual
    case); only elements near a rounding tie get a nonzero bound.  Computed
    from oracle quantities only."""
    x = np.asarray(x_ref, np.float64)
    M, K = x.shape
    xb = x.reshape(M, K // 32, 32)
    tb = np.asarray(x_tol, np.float64).reshape(M, K // 32, 32)
    T = tb.max(axis=2)
    amax = np.abs(xb).max(axis=2)
    ulp32 = 2.0 ** -23
    d32_lo = np.maximum(amax - T, 0) / 127 * (1 - 2 * ulp32)
    d32_hi = (amax + T) / 127 * (1 + 2 * ulp32)
    fp16 = o.fp16_values()
    d_lo = fp16[o.fp32_to_fp16_bits(d32_lo.astype(np.float32))]
    d_hi = fp16[o.fp32_to_fp16_bits(d32_hi.astype(np.float32))]
    # the oracle's own quantisation of x_ref: the activations it multiplies
    q_o, d_o = o.quantize_q8_0(np.asarray(x_ref, np.float32))
    a_ref = (fp16[d_o][..., None] * q_o.reshape(M, K // 32, 32).astype(np.float64))
    with np.errstate(divide="ignore", invalid="ignore"):
        r_a = (xb - tb) / d32_lo[..., None]
        r_b = (xb + tb) / d32_lo[..., None]
        r_c = (xb - tb) / d32_hi[..., None]
        r_d = (xb + tb) / d32_hi[..., None]
    rs = np.stack([r_a, r_b, r_c, r_d])
    rs = np.where(np.isfinite(rs), rs, 0.0)
    q_lo = np.clip(np.rint(rs.min(axis=0) - 1e-6), -127, 127)
    q_hi = np.clip(np.rint(rs.max(axis=0) + 1e-6), -127, 127)
    cand = [d_lo[..., None] * q_lo, d_lo[..., None] * q_hi,
            d_hi[..., None] * q_lo, d_hi[..., None] * q_hi]
    bound = np.max([np.abs(c - a_ref) for c in cand], axis=0)
    return bound.reshape(M, K)


def chained_reference(P: Packed, x_ref: np.ndarray, da: np.ndarray):
    """Oracle output of one product whose input activations come from a
    requantisation with per-element uncertainty da (zeros for exact inputs):
    returns (y_ref fp64, tol) with tol = the usual bound on the larger
    sum|terms| plus sum_k |w[n, k]| * da[m, k]."""
    q_ref, d_ref = o.quantize_q8_0(x_ref.astype(np.float32))
    y, sa, _ = reference(P, q_ref, d_ref)
    if np.any(da > 0):
        w_abs = np.abs(o.dequantize_weights(P.ref_codes, P.ref_scales, P.ref_g))
        spread = da @ w_abs.T
    else:
        spread = np.zeros_like(y)
    tol = o.tolerance(sa + spread) + spread
    return y, tol
