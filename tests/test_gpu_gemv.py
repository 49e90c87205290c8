"""GPU parity of the decode GEMV (M = 1..16) and of its integer subblock sums.

* small shapes the oracle finishes in seconds, spanning several CTAs, a
  ragged row count (not a multiple of the rows per stage or CTA) and ragged
  chunk counts per lane: every output element compared;
* every M = 1 kernel instantiation the dispatch can pick (register schedule
  for each (chunks per lane, warps per row) pair, the shared-memory schedule
  for segments of 5120, 4096 and other sizes, the TMA schedule and the plain
  one-warp-per-row kernel);
* the full decode-sweep and small-batch shapes: every row computed on the
  GPU, a sample of rows checked against the oracle;
* integer subblock sums: exported by nvq_debug_subblock_sums, which runs
  the same dispatch and kernels as nvq_gemv instantiated to store them, and
  compared bit for bit (int32 vs the oracle's int64); the y it writes is
  bit-identical to nvq_gemv's;
* fp32 outputs: |y - y_ref| <= 1e-5 * sum|terms| + 1e-6 per element.
"""
import numpy as np
import pytest
import torch

from bit_weight_quantized_nvq_b200 import capi, workloads as wl
from parity import Packed, assert_within_tolerance, quantize_both, reference, sample_rows

pytestmark = pytest.mark.gpu


def run_gemv(P, q, d):
    y = capi.gemv(P.codes, P.scales, P.g, q, d)
    torch.cuda.synchronize()
    return y


def check_isums(P, q, d, y_gemv, isum_ref, rows=None):
    """Integer sums of the GEMV's own kernels: bit-exact against the oracle;
    the y of that launch equals nvq_gemv's bit for bit."""
    y_dbg, isum = capi.debug_subblock_sums(P.codes, P.scales, P.g, q, d)
    torch.cuda.synchronize()
    assert torch.equal(y_dbg, y_gemv), "the integer-sum instantiation changed y"
    got = isum.cpu().numpy()
    if rows is not None:
        got = got[:, rows]
    assert np.array_equal(got.astype(np.int64), isum_ref)


# (1001, 1088), (37, 64), (1, 4160): K % 256 != 0, the one-warp-per-row kernel.
# (1001, 1280): shared-memory / TMA schedules, one K segment, ragged row groups.
# (37, 12800): K segments of 2560 per row.
# (300, 25600): the decode K with few rows (one or two rows per CTA).
@pytest.mark.parametrize("M", list(range(1, 17)))
@pytest.mark.parametrize("N,K", [(1001, 1088), (37, 64), (1, 4096 + 64),
                                 (1001, 1280), (37, 12800), (300, 25600)])
def test_small_shapes_all_rows(M, N, K):
    W = wl.weights("gemv_test", "W", N, K, boost_columns=True)
    x = wl.activations("gemv_test", "x", M, K, "student_t4")
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemv(P, q, d)
    y_ref, sa, isum_ref = reference(P, q_ref, d_ref)
    assert_within_tolerance(y.cpu().numpy(), y_ref, sa)
    check_isums(P, q, d, y, isum_ref)


# K -> the M = 1 kernel nvq_gemv dispatches to:
#   K = 1024*T, T in {2,3,4,5,6,8,10,12,15,16,20,25}: register schedule
#     <chunks per lane, warps per row> = <2,1> <3,1> <4,1> <5,1> <6,1> <4,2> <5,2> <6,2>
#     <5,3> <4,4> <5,4> <5,5>;
#   30720: shared-memory schedule, 5120-element segments (<5>);
#   28672: shared-memory schedule, 4096-element segments (<4>);
#   1280, 12800: shared-memory schedule, other segments (<0>);
#   35840: its shared memory does not fit, the TMA schedule <1>;
#   1088: K % 256 != 0, the one-warp-per-row kernel <1>.
M1_DISPATCH_KS = [2048, 3072, 4096, 5120, 6144, 8192, 10240, 12288, 15360, 16384, 20480, 25600,
                  30720, 28672, 1280, 12800, 35840, 1088]


@pytest.mark.parametrize("K", M1_DISPATCH_KS)
def test_every_m1_instantiation_bit_exact_sums(K):
    N = 333                                        # a few rows per CTA, ragged stages
    W = wl.weights("gemv_test", "Wm1", N, K, boost_columns=True)
    x = wl.activations("gemv_test", "xm1", 1, K, "student_t4")
    x[0, 64:96] = 0.0                              # a zero block (d = 0, corr = 0)
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemv(P, q, d)
    y_ref, sa, isum_ref = reference(P, q_ref, d_ref)
    assert_within_tolerance(y.cpu().numpy(), y_ref, sa)
    check_isums(P, q, d, y, isum_ref)


def test_gemv_4096_all_rows():
    W, x = wl.gemv_4096_case()
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemv(P, q, d)
    y_ref, sa, isum_ref = reference(P, q_ref, d_ref)
    assert_within_tolerance(y.cpu().numpy(), y_ref, sa)
    check_isums(P, q, d, y, isum_ref)


@pytest.mark.parametrize("K,N", wl.DECODE_SHAPES)
def test_decode_sweep_full_size_sampled(K, N):
    W, x = wl.decode_case(K, N)
    rows = sample_rows(N, 384, seed=K + N)
    P = Packed(W, rows)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemv(P, q, d)
    y_ref, sa, isum_ref = reference(P, q_ref, d_ref)
    assert_within_tolerance(y.cpu().numpy()[:, rows], y_ref, sa)
    check_isums(P, q, d, y, isum_ref, rows)


@pytest.mark.parametrize("M", wl.SMALL_BATCH_MS)
@pytest.mark.parametrize("K,N", wl.SMALL_BATCH_SHAPES)
def test_small_batch_full_size_sampled(M, K, N):
    W, x = wl.small_batch_case(M, K, N)
    rows = sample_rows(N, 256, seed=M + K + N)
    P = Packed(W, rows)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemv(P, q, d)
    y_ref, sa, isum_ref = reference(P, q_ref, d_ref)
    assert_within_tolerance(y.cpu().numpy()[:, rows], y_ref, sa)
    check_isums(P, q, d, y, isum_ref, rows)


def test_degenerate_inputs():
    K, N = 256, 64
    W = wl.weights("gemv_test", "W", N, K)
    W[5] = 0.0                                     # an all-zero row (scales 0)
    W[6, :16] = 1e-12                              # a subnormal-scale subblock
    x = wl.activations("gemv_test", "x", 2, K, "normal")
    x[1, :] = 0.0                                  # an all-zero token (d = 0)
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    y = run_gemv(P, q, d).cpu().numpy()
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    assert_within_tolerance(y, y_ref, sa)
    assert np.all(y[1] == 0) and np.all(y[:, 5] == 0)
    # zero scales give exactly zero everywhere
    y0 = capi.gemv(P.codes, torch.zeros_like(P.scales), P.g, q, d)
    torch.cuda.synchronize()
    assert not y0.cpu().numpy().any()


@pytest.mark.parametrize("M,K", [(1, 5120), (1, 1280), (3, 512)])
def test_sign_flip_of_a_subblock_negates_its_integer_sum(M, K):
    N = 16
    W = wl.weights("gemv_test", "W", N, K)
    x = wl.activations("gemv_test", "x", M, K, "normal")
    P = Packed(W)
    q, d, _, _ = quantize_both(x)
    _, base = capi.debug_subblock_sums(P.codes, P.scales, P.g, q, d)
    flipped = P.codes.clone()
    flipped[3, 8 * 7:8 * 8] ^= 0x88                # subblock 7 of row 3
    _, f = capi.debug_subblock_sums(flipped, P.scales, P.g, q, d)
    base, f = base.cpu().numpy(), f.cpu().numpy()
    assert np.array_equal(f[:, 3, 7], -base[:, 3, 7])
    mask = np.ones_like(base, bool)
    mask[:, 3, 7] = False
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
    with pytest.raises(capi.NVQError) as e:
        capi.debug_subblock_sums(codes, scales, 1.0, q, d)
    assert e.value.status == capi.NVQ_ERR_BAD_SHAPE
