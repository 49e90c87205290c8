"""GPU parity of the NVFP4 x NVFP4 path: the NVFP4 activation quantiser
(nvq_quantize_act_nvfp4) and the block-scaled FP4 tensor-core GEMM
(nvq_gemm_nvf4).

* the quantiser's codes, scales and per-token g equal the oracle's
  quantize_act_nvfp4 bit for bit: ragged K (K % 256 != 0), zero tokens,
  tokens with one huge channel, subnormal-range values, exact rounding ties
  of the E2M1 grid;
* the GEMM on shapes the oracle finishes in seconds, every element compared:
  one 128-token tile and several, ragged weight rows and tokens (not a
  multiple of the 128-row tile), one K stage and K long enough to use both
  accumulator buffers several times; and the 256-token tiles (single
  accumulator promoted every 4096 K) on sampled rows;
* the prefill shapes at full size, sampled weight rows and tokens;
* zero scales give zero, a zero token gives a zero row, repeated calls are
  bit-identical, bad shapes are refused before any launch;
* fp32 outputs: |y - y_ref| <= 1e-5 * sum_k |w*a| + 1e-6 per element.
"""
import numpy as np
import pytest
import torch

import oracle as o
from bit_weight_quantized_nvq_b200 import capi, workloads as wl
from parity import assert_within_tolerance, sample_rows, to_dev

pytestmark = pytest.mark.gpu


def quantize_nvf4_both(x: np.ndarray):
    """GPU and oracle NVFP4 activations of x; asserts they are bit-identical."""
    codes, scales, g = capi.quantize_act_nvfp4(to_dev(x))
    torch.cuda.synchronize()
    rc, rs, rg = o.quantize_act_nvfp4(x)
    assert np.array_equal(codes.cpu().numpy(), rc), "NVFP4 activation codes differ"
    assert np.array_equal(scales.cpu().numpy(), rs), "NVFP4 activation scales differ"
    assert np.array_equal(g.cpu().numpy().view(np.uint32), rg.view(np.uint32)), "token scales differ"
    return (codes, scales, g), (rc, rs, rg)


def pack_weights(W: np.ndarray):
    codes, scales, g = capi.pack_nvfp4(W)
    rc, rs, rg = o.pack_nvfp4(W)
    assert np.float32(g) == rg and np.array_equal(codes, rc) and np.array_equal(scales, rs)
    return (to_dev(codes), to_dev(scales), g), (rc, rs, rg)


def reference(wref, aref, rows=None, toks=None):
    wc, ws, wg = wref
    ac, as_, ag = aref
    if rows is not None:
        wc, ws = wc[rows], ws[rows]
    if toks is not None:
        ac, as_, ag = ac[toks], as_[toks], ag[toks]
    return (o.dot_fp64_nvf4(wc, ws, wg, ac, as_, ag),
            o.sum_abs_terms_nvf4(wc, ws, wg, ac, as_, ag))


# K -> schedule: one CTA per row up to 256 subblocks (16 .. 4096), a cluster
# of 2..8 CTAs per row up to 2048 (5120, 25600), the two-pass kernel beyond
# (33024).
@pytest.mark.parametrize("M,K", [(1, 16), (3, 272), (37, 4096), (300, 5120), (5, 25600),
                                 (3, 33024)])
def test_quantiser_bit_exact(M, K):
    x = wl.activations("nvf4_test", "xq", M, K, "student_t4", outliers=K >= 1024)
    if M >= 3:
        x[1] = 0.0                               # an all-zero token: g = 0, codes 0
        x[2, :] *= np.float32(1e-38)             # values in the fp32 subnormal range
    quantize_nvf4_both(x)


def test_quantiser_rounding_ties_and_saturation():
    # amax 6 in every subblock: g = 6/2688, s = UE4M3(1) = 1.0, x/(g*s) = x*448
    # lands on exact E2M1 midpoints (0.25, 0.75, ..., 5) and beyond 6.
    K = 64
    grid = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 5.5, -0.25, -2.5, -5.0, 0.0,
                     -0.0, 0.1, 4.0, 6.0], np.float32)
    g = np.float32(6.0) / np.float32(2688.0)
    x = np.tile(grid, K // 16)[None, :] * g
    x = np.concatenate([x, -x, x * np.float32(3.7)], axis=0).astype(np.float32)
    quantize_nvf4_both(x)


# (M, N, K): one stage; one 128x128 tile exactly; ragged rows and tokens over
# several tiles; 20 stages (five 1024-K chunks, both accumulators reused);
# a single token; 257 tokens = three token tiles.
@pytest.mark.parametrize("M,N,K", [
    (1, 37, 256), (128, 128, 256), (130, 300, 1280), (5, 129, 512), (200, 257, 5120),
    (257, 64, 2048), (64, 1000, 4096), (16, 520, 25600),
])
def test_gemm_all_elements(M, N, K):
    W = wl.weights("nvf4_test", "W", N, K, boost_columns=True)
    x = wl.activations("nvf4_test", "x", M, K, "student_t4", outliers=True)
    (wc, ws, wg), wref = pack_weights(W)
    (ac, as_, ag), aref = quantize_nvf4_both(x)
    y = capi.gemm_nvf4(wc, ws, wg, ac, as_, ag)
    torch.cuda.synchronize()
    y_ref, sa = reference(wref, aref)
    assert_within_tolerance(y.cpu().numpy(), y_ref, sa)
    assert capi.error_flags() == 0


# 256-token tiles (chosen when they still fill every SM twice: here 2 token
# tiles x 149 weight tiles): a full tile and a ragged one (300 tokens), one
# K stage and K = 4352 (two chunks of the single accumulator: 16 + 1 stages).
@pytest.mark.parametrize("M,N,K", [(512, 19000, 256), (300, 19000, 4352)])
def test_gemm_256_token_tiles_sampled_rows(M, N, K):
    W = wl.weights("nvf4_test", "W256", N, K)
    x = wl.activations("nvf4_test", "x256", M, K, "student_t4", outliers=True)
    codes, scales, g = capi.pack_nvfp4(W)
    rows = sample_rows(N, 96, seed=M + N + K)
    wref = o.pack_nvfp4(W[rows], g=o.nvfp4_tensor_scale(W))
    assert np.array_equal(codes[rows], wref[0]) and np.array_equal(scales[rows], wref[1])
    (ac, as_, ag), aref = quantize_nvf4_both(x)
    y = capi.gemm_nvf4(to_dev(codes), to_dev(scales), g, ac, as_, ag)
    torch.cuda.synchronize()
    y_ref, sa = reference(wref, aref)
    assert_within_tolerance(y.cpu().numpy()[:, rows], y_ref, sa)
    assert capi.error_flags() == 0


@pytest.mark.parametrize("M", wl.PREFILL_MS)
@pytest.mark.parametrize("K,N", wl.PREFILL_SHAPES)
def test_prefill_full_size_sampled(M, K, N):
    W, x = wl.prefill_case(M, K, N)
    codes, scales, g = capi.pack_nvfp4(W)
    rows = sample_rows(N, 96, seed=M + K + N + 7)
    toks = sample_rows(M, 24, seed=M + K + N + 8)
    wref = o.pack_nvfp4(W[rows], g=o.nvfp4_tensor_scale(W))
    assert np.float32(g) == wref[2]
    assert np.array_equal(codes[rows], wref[0]) and np.array_equal(scales[rows], wref[1])
    ac, as_, ag = capi.quantize_act_nvfp4(to_dev(x))
    y = capi.gemm_nvf4(to_dev(codes), to_dev(scales), g, ac, as_, ag)
    torch.cuda.synchronize()
    aref = o.quantize_act_nvfp4(x[toks])
    assert np.array_equal(ac.cpu().numpy()[toks], aref[0])
    assert np.array_equal(as_.cpu().numpy()[toks], aref[1])
    assert np.array_equal(ag.cpu().numpy()[toks], aref[2])
    y_ref, sa = reference(wref, aref)
    y_h = y.cpu().numpy()
    assert np.all(np.isfinite(y_h))
    assert_within_tolerance(y_h[np.ix_(toks, rows)], y_ref, sa)


def test_zero_scales_zero_tokens_and_determinism():
    M, N, K = 150, 300, 1024
    W = wl.weights("nvf4_test", "Wz", N, K)
    x = wl.activations("nvf4_test", "xz", M, K, "normal")
    x[7] = 0.0
    (wc, ws, wg), wref = pack_weights(W)
    (ac, as_, ag), aref = quantize_nvf4_both(x)
    y1 = capi.gemm_nvf4(wc, ws, wg, ac, as_, ag)
    y2 = capi.gemm_nvf4(wc, ws, wg, ac, as_, ag)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    y_h = y1.cpu().numpy()
    assert not y_h[7].any()
    y_ref, sa = reference(wref, aref)
    assert_within_tolerance(y_h, y_ref, sa)
    y0 = capi.gemm_nvf4(wc, torch.zeros_like(ws), wg, ac, as_, ag)
    torch.cuda.synchronize()
    assert not y0.cpu().numpy().any()


def test_bad_shapes_are_refused():
    dev = "cuda"
    wc = torch.zeros((64, 64), dtype=torch.uint8, device=dev)      # K = 128: K % 256 != 0
    ws = torch.zeros((64, 8), dtype=torch.uint8, device=dev)
    ac = torch.zeros((4, 64), dtype=torch.uint8, device=dev)
    as_ = torch.zeros((4, 8), dtype=torch.uint8, device=dev)
    ag = torch.zeros((4,), dtype=torch.float32, device=dev)
    with pytest.raises(capi.NVQError) as e:
        capi.gemm_nvf4(wc, ws, 1.0, ac, as_, ag)
    assert e.value.status == capi.NVQ_ERR_BAD_SHAPE
    with pytest.raises(capi.NVQError) as e:
        capi.quantize_act_nvfp4(torch.zeros((2, 24), dtype=torch.float32, device=dev))
    assert e.value.status == capi.NVQ_ERR_BAD_SHAPE
