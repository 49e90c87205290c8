"""GPU parity of the tcgen05 prefill GEMM.

* small and ragged shapes (M and N not multiples of the 128 x 128 tile, K a
  single 64-block up to 25600): every output element compared;
* the full prefill shapes (M in {256, 2048}; (K, N) = (5120, 5120),
  (5120, 25600), (25600, 5120)): every element computed, a sample of rows and
  tokens checked against the oracle;
* stream-K tails (the tiles of the last partial wave split over every CTA
  pair): one tile in up to 74 parts, fewer leftover K stages than pairs,
  a ragged last K stage; the split tiles' rows and tokens are checked;
* tokens whose activations exceed the fp16 range (the 2^-e pre-scale);
* fp32 outputs: |y - y_ref| <= 1e-5 * sum|terms| + 1e-6 per element.
"""
import numpy as np
import pytest
import torch

import oracle as o
from bit_weight_quantized_nvq_b200 import capi, workloads as wl
from parity import Packed, assert_within_tolerance, quantize_both, reference, sample_rows

pytestmark = pytest.mark.gpu


def run_gemm(P, q, d):
    y = capi.gemm(P.codes, P.scales, P.g, q, d)
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("M,N,K", [
    (1, 37, 64), (5, 128, 128), (17, 129, 192), (128, 256, 512), (130, 300, 1088),
    (300, 520, 4096), (257, 200, 25600), (64, 1000, 5120),
])
def test_small_shapes_all_elements(M, N, K):
    W = wl.weights("gemm_test", "W", N, K, boost_columns=True)
    x = wl.activations("gemm_test", "x", M, K, "normal", outliers=True)
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemm(P, q, d)
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    assert_within_tolerance(y, y_ref, sa)


@pytest.mark.parametrize("M", wl.PREFILL_MS)
@pytest.mark.parametrize("K,N", wl.PREFILL_SHAPES)
def test_prefill_full_size_sampled(M, K, N):
    W, x = wl.prefill_case(M, K, N)
    rows = sample_rows(N, 96, seed=M + K + N)
    P = Packed(W, rows)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemm(P, q, d)
    toks = sample_rows(M, 192, seed=M * 7 + K)
    y_ref, sa, _ = reference(P, q_ref[toks], d_ref[toks])
    assert_within_tolerance(y[np.ix_(toks, rows)], y_ref, sa)
    assert np.all(np.isfinite(y))


# The persistent GEMM gives each of the CTA pairs (74 on a 148-SM B200) whole
# tiles of 128 tokens x 256 weight rows round-robin and splits the K stages
# of the tiles left over evenly.  With 300 tokens and 6400 rows there are
# 3 x 25 = 75 tiles (token tiles run fastest here): one left over, the tile
# of tokens 256..299 and rows 6144..6399.  At K = 25600 its 200 stages go to
# all 74 pairs (2-3 each); at K = 1024 its 8 stages go to 8 pairs, the others
# getting none.  With (130, 5184, 300) all 4 tiles are split, each of 41
# stages whose last is 64 wide.
@pytest.mark.parametrize("M,K,N,tail", [
    (300, 25600, 6400, True), (300, 1024, 6400, True), (130, 5184, 300, False),
])
def test_stream_k_tails_sampled(M, K, N, tail):
    W = wl.weights("gemm_test", "Wsk", N, K, boost_columns=True)
    x = wl.activations("gemm_test", "xsk", M, K, "normal", outliers=True)
    if tail:
        rows = np.union1d(sample_rows(N, 32, seed=K), np.arange(6144, 6400, 3))
        toks = np.union1d(sample_rows(M, 16, seed=K + 1), np.arange(256, 300))
    else:
        rows, toks = np.arange(N), np.arange(M)
    P = Packed(W, rows)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemm(P, q, d)
    y_ref, sa, _ = reference(P, q_ref[toks], d_ref[toks])
    assert_within_tolerance(y[np.ix_(toks, rows)], y_ref, sa)
    assert np.all(np.isfinite(y))


def test_activations_beyond_fp16_range():
    M, N, K = 6, 256, 1024
    W = wl.weights("gemm_test", "W", N, K)
    x = wl.activations("gemm_test", "x", M, K, "normal")
    x[1] *= 1e5                     # |x| up to ~4e5: d*q beyond 65504
    x[2, :64] = 3e6                 # d near the fp16 maximum
    x[3, :32] = 1e-3                # tiny blocks in an otherwise normal token
    x[3, 32:] *= 2e4
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemm(P, q, d)
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    assert_within_tolerance(y, y_ref, sa)


def test_gemm_agrees_with_gemv_for_small_m():
    M, N, K = 16, 1024, 5120
    W, x = wl.small_batch_case(M, K, 25600)
    W = np.ascontiguousarray(W[:N])
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    y_mm = run_gemm(P, q, d)
    y_mv = capi.gemv(P.codes, P.scales, P.g, q, d).cpu().numpy()
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    assert_within_tolerance(y_mm, y_ref, sa)
    assert_within_tolerance(y_mv, y_ref, sa)


def test_zero_scales_and_zero_tokens():
    M, N, K = 130, 140, 256
    W = wl.weights("gemm_test", "W", N, K)
    x = wl.activations("gemm_test", "x", M, K, "normal")
    x[7] = 0.0
    P = Packed(W)
    q, d, _, _ = quantize_both(x)
    y = run_gemm(P, q, d)
    assert np.all(y[7] == 0)
    y0 = capi.gemm(P.codes, torch.zeros_like(P.scales), P.g, q, d)
    torch.cuda.synchronize()
    assert not y0.cpu().numpy().any()


def test_workspace_reuse_and_error_status():
    M, N, K = 40, 64, 128
    W = wl.weights("gemm_test", "W", N, K)
    x = wl.activations("gemm_test", "x", M, K, "normal")
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    ws = torch.full((capi.gemm_workspace_size(M, N, K),), 0xAB, dtype=torch.uint8, device="cuda")
    y1 = capi.gemm(P.codes, P.scales, P.g, q, d, workspace=ws).cpu().numpy()
    y2 = capi.gemm(P.codes, P.scales, P.g, q, d, workspace=ws).cpu().numpy()
    assert np.array_equal(y1, y2)
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    assert_within_tolerance(y1, y_ref, sa)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(capi.NVQError) as e:
        capi.gemm(P.codes, P.scales, P.g, q, d, workspace=small)
    assert e.value.status == capi.NVQ_ERR_WORKSPACE
