"""GPU parity of the decode GEMV (M = 1..16) and of its integer subblock sums.

* small shapes the oracle finishes in seconds, spanning several CTAs, a
  ragged row count (not a multiple of the four rows per CTA) and ragged
  chunk counts per lane: every output element compared;
* the full decode-sweep and small-batch shapes: every row computed on the
  GPU, a sample of rows checked against the oracle;
* integer subblock sums: bit-exact (int32 vs int64);
* fp32 outputs: |y - y_ref| <= 1e-5 * sum|terms| + 1e-6 per element.
"""
import numpy as np
import pytest
import torch

import oracle as o
from bit_weight_quantized_nvq_b200 import capi, workloads as wl
from parity import Packed, assert_within_tolerance, quantize_both, reference, sample_rows

pytestmark = pytest.mark.gpu


def run_gemv(P, q, d, M):
    y = capi.gemv(P.codes, P.scales, P.g, q, d)
    torch.cuda.synchronize()
    return y.cpu().numpy()


# (1001, 1088), (37, 64), (1, 4160): K % 256 != 0, the register schedule.
# (1001, 1280): the TMA schedule, one K segment, ragged row groups.
# (37, 12800): the TMA schedule with five K segments of 2560 per row.
# (300, 25600): the decode K with few rows (one or two rows per CTA).
@pytest.mark.parametrize("M", list(range(1, 17)))
@pytest.mark.parametrize("N,K", [(1001, 1088), (37, 64), (1, 4096 + 64),
                                 (1001, 1280), (37, 12800), (300, 25600)])
def test_small_shapes_all_rows(M, N, K):
    W = wl.weights("gemv_test", "W", N, K, boost_columns=True)
    x = wl.activations("gemv_test", "x", M, K, "student_t4")
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemv(P, q, d, M)
    y_ref, sa, isum_ref = reference(P, q_ref, d_ref)
    assert_within_tolerance(y, y_ref, sa)
    isum = capi.debug_subblock_sums(P.codes, q)
    torch.cuda.synchronize()
    assert np.array_equal(isum.cpu().numpy().astype(np.int64), isum_ref)


def test_gemv_4096_all_rows():
    W, x = wl.gemv_4096_case()
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemv(P, q, d, 1)
    y_ref, sa, isum_ref = reference(P, q_ref, d_ref)
    assert_within_tolerance(y, y_ref, sa)
    isum = capi.debug_subblock_sums(P.codes, q)
    torch.cuda.synchronize()
    assert np.array_equal(isum.cpu().numpy().astype(np.int64), isum_ref)


@pytest.mark.parametrize("K,N", wl.DECODE_SHAPES)
def test_decode_sweep_full_size_sampled(K, N):
    W, x = wl.decode_case(K, N)
    rows = sample_rows(N, 384, seed=K + N)
    P = Packed(W, rows)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemv(P, q, d, 1)
    y_ref, sa, isum_ref = reference(P, q_ref, d_ref)
    assert_within_tolerance(y[:, rows], y_ref, sa)
    isum = capi.debug_subblock_sums(P.codes, q)
    torch.cuda.synchronize()
    assert np.array_equal(isum.cpu().numpy()[:, rows].astype(np.int64), isum_ref)


@pytest.mark.parametrize("M", wl.SMALL_BATCH_MS)
@pytest.mark.parametrize("K,N", wl.SMALL_BATCH_SHAPES)
def test_small_batch_full_size_sampled(M, K, N):
    W, x = wl.small_batch_case(M, K, N)
    rows = sample_rows(N, 256, seed=M + K + N)
    P = Packed(W, rows)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemv(P, q, d, M)
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    assert_within_tolerance(y[:, rows], y_ref, sa)


def test_degenerate_inputs():
    K, N = 256, 64
    W = wl.weights("gemv_test", "W", N, K)
    W[5] = 0.0                                     # an all-zero row (scales 0)
    W[6, :16] = 1e-12                              # a subnormal-scale subblock
    x = wl.activations("gemv_test", "x", 2, K, "normal")
    x[1, :] = 0.0                                  # an all-zero token (d = 0)
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemv(P, q, d, 2)
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    assert_within_tolerance(y, y_ref, sa)
    assert np.all(y[1] == 0) and np.all(y[:, 5] == 0)
    # zero scales give exactly zero everywhere
    y0 = capi.gemv(P.codes, torch.zeros_like(P.scales), P.g, q, d)
    torch.cuda.synchronize()
    assert not y0.cpu().numpy().any()


def test_sign_flip_of_a_subblock_negates_its_integer_sum():
    K, N = 512, 16
    W = wl.weights("gemv_test", "W", N, K)
    x = wl.activations("gemv_test", "x", 1, K, "normal")
    P = Packed(W)
    q, d, _, _ = quantize_both(x)
    base = capi.debug_subblock_sums(P.codes, q).cpu().numpy()
    flipped = P.codes.clone()
    flipped[3, 8 * 7:8 * 8] ^= 0x88                # subblock 7 of row 3
    f = capi.debug_subblock_sums(flipped, q).cpu().numpy()
    assert np.array_equal(f[0, 3, 7], -base[0, 3, 7])
    mask = np.ones_like(base, bool)
    mask[0, 3, 7] = False
    assert np.array_equal(f[mask], base[mask])


def test_empty_product_launches_nothing():
    codes = torch.zeros((0, 32), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((0, 4), dtype=torch.uint8, device="cuda")
    q = torch.zeros((1, 64), dtype=torch.int8, device="cuda")
    d = torch.zeros((1, 2), dtype=torch.float16, device="cuda")
    y = capi.gemv(codes, scales, 1.0, q, d)
    assert y.shape == (1, 0)


def test_error_status_on_device():
    q = torch.zeros((17, 64), dtype=torch.int8, device="cuda")
    d = torch.zeros((17, 2), dtype=torch.float16, device="cuda")
    codes = torch.zeros((4, 32), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((4, 4), dtype=torch.uint8, device="cuda")
    with pytest.raises(capi.NVQError) as e:
        capi.gemv(codes, scales, 1.0, q, d)
    assert e.value.status == capi.NVQ_ERR_BAD_SHAPE


@pytest.mark.parametrize("K,N", [(4096, 1000), (5120, 1537), (25600, 700), (10240, 301),
                                 (6144, 257), (5120, 152064)])
def test_fused_quant_gemv_is_bit_identical_and_within_tolerance(K, N):
    W = wl.weights("gemv_test", "Wf", N, K, boost_columns=True)
    x = wl.activations("gemv_test", "xf", 1, K, "student_t4")
    x[0, :32] = 0.0                               # a zero block (d = 0)
    rows = sample_rows(N, 300, seed=K + N) if N > 2000 else None
    P = Packed(W, rows)
    xd = torch.from_numpy(x).cuda()
    y_f = capi.quant_gemv(P.codes, P.scales, P.g, xd)
    q, d = capi.quantize_act_q8_0(xd)
    y_u = capi.gemv(P.codes, P.scales, P.g, q, d)
    torch.cuda.synchronize()
    assert torch.equal(y_f, y_u)
    q_ref, d_ref = o.quantize_q8_0(x)
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    y = y_f.cpu().numpy()
    assert_within_tolerance(y if rows is None else y[:, rows], y_ref, sa)


def test_fused_quant_gemv_rejects_unsupported_k():
    codes = torch.zeros((4, 1088 // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((4, 1088 // 16), dtype=torch.uint8, device="cuda")
    x = torch.zeros((1, 1088), device="cuda")
    with pytest.raises(capi.NVQError) as e:
        capi.quant_gemv(codes, scales, 1.0, x)
    assert e.value.status == capi.NVQ_ERR_BAD_SHAPE
