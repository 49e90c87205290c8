"""GPU parity of nvq_gemm at M = 1..16: M <= 4 runs the decode GEMV, 5..16
(K % 256 == 0) the small-token tensor-core schedule: weights expanded into
tensor memory, the exact fp16 hi/lo
activations by TMA, tcgen05.mma with fp32 accumulation promoted every
1024 K, and the work split in equal ranges of (row tile, K stage) units over
the SMs (stream-K), with split tiles added in a fixed order.

* shapes the oracle finishes in seconds, every element compared: ragged
  row counts (not a multiple of the 128-row tile), one-stage and many-stage
  K, tiles split between many CTAs and tiles owned by one, 1..16 tokens;
* the small-batch workload shapes at full size, sampled rows;
* determinism (a split tile is summed in a fixed order), zero scales and
  zero tokens, and tokens whose activations exceed the fp16 range;
* fp32 outputs: |y - y_ref| <= 1e-5 * sum|terms| + 1e-6 per element.
"""
import numpy as np
import pytest
import torch

from bit_weight_quantized_nvq_b200 import capi, workloads as wl
from parity import Packed, assert_within_tolerance, quantize_both, reference, sample_rows

pytestmark = pytest.mark.gpu


def run_gemm(P, q, d):
    y = capi.gemm(P.codes, P.scales, P.g, q, d)
    torch.cuda.synchronize()
    return y.cpu().numpy()


# (M, N, K): 37 rows / one stage; 129 rows = two tiles; 1000 rows x 20 stages
# over 148 SMs (each tile split between ~18 CTAs); 300 rows x 5 stages;
# 128 rows exactly; 16 tokens x 100 stages (K = 25600) on 520 rows.
@pytest.mark.parametrize("M,N,K", [
    (1, 37, 256), (2, 129, 512), (3, 1000, 5120), (5, 300, 1280), (8, 128, 256),
    (9, 200, 2560), (12, 1001, 4096), (16, 520, 25600), (16, 1, 256), (7, 2048, 1024),
    (4, 25600 // 16, 5120), (13, 640, 12288),
])
def test_small_token_shapes_all_elements(M, N, K):
    W = wl.weights("gemm_small_test", "W", N, K, boost_columns=True)
    x = wl.activations("gemm_small_test", "x", M, K, "student_t4")
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemm(P, q, d)
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    assert_within_tolerance(y, y_ref, sa)


@pytest.mark.parametrize("M", wl.SMALL_BATCH_MS)
@pytest.mark.parametrize("K,N", wl.SMALL_BATCH_SHAPES)
def test_small_batch_full_size_sampled(M, K, N):
    W, x = wl.small_batch_case(M, K, N)
    rows = sample_rows(N, 256, seed=M + K + N + 1)
    P = Packed(W, rows)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemm(P, q, d)
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    assert_within_tolerance(y[:, rows], y_ref, sa)
    assert np.all(np.isfinite(y))


def test_deterministic_and_agrees_with_the_gemv():
    M, N, K = 6, 3000, 5120
    W = wl.weights("gemm_small_test", "Wd", N, K, boost_columns=True)
    x = wl.activations("gemm_small_test", "xd", M, K, "student_t4")
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    y1 = run_gemm(P, q, d)
    y2 = run_gemm(P, q, d)
    assert np.array_equal(y1, y2), "split tiles must be added in a fixed order"
    y_mv = capi.gemv(P.codes, P.scales, P.g, q, d).cpu().numpy()
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    assert_within_tolerance(y1, y_ref, sa)
    assert_within_tolerance(y_mv, y_ref, sa)


def test_zero_scales_zero_tokens_and_fp16_overflow():
    M, N, K = 6, 300, 1024
    W = wl.weights("gemm_small_test", "Wz", N, K)
    x = wl.activations("gemm_small_test", "xz", M, K, "normal")
    x[2] = 0.0                       # an all-zero token (d = 0)
    x[1] *= 1e5                      # |d*q| beyond 65504: the 2^-e token pre-scale
    x[4, :64] = 3e6
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemm(P, q, d)
    assert np.all(y[2] == 0)
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    assert_within_tolerance(y, y_ref, sa)
    y0 = capi.gemm(P.codes, torch.zeros_like(P.scales), P.g, q, d)
    torch.cuda.synchronize()
    assert not y0.cpu().numpy().any()


def test_workspace_size_and_reuse():
    M, N, K = 16, 700, 2048
    need = capi.gemm_workspace_size(M, N, K)
    assert need >= 4 * 16 * K                     # the hi/lo expansion of 16 padded tokens
    W = wl.weights("gemm_small_test", "Ww", N, K)
    x = wl.activations("gemm_small_test", "xw", M, K, "normal")
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    ws = torch.full((need,), 0xAB, dtype=torch.uint8, device="cuda")
    y1 = capi.gemm(P.codes, P.scales, P.g, q, d, workspace=ws).cpu().numpy()
    y2 = capi.gemm(P.codes, P.scales, P.g, q, d, workspace=ws).cpu().numpy()
    assert np.array_equal(y1, y2)
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    assert_within_tolerance(y1, y_ref, sa)
    with pytest.raises(capi.NVQError) as e:
        capi.gemm(P.codes, P.scales, P.g, q, d, workspace=ws[:need - 1])
    assert e.value.status == capi.NVQ_ERR_WORKSPACE
    assert capi.error_flags() == 0
