"""GPU parity of the fused requantisation epilogue (nvq_gemv_requant) and of
the grouped GEMV (nvq_gemv_grouped).

* the GEMV's y is within the fp32 tolerance of the oracle, and the emitted
  Q8_0 codes and fp16 scales equal the oracle's quantisation of that very y
  bit for bit (the block is quantised by whichever CTA completes it);
* the block counters are back at zero after every call, so a second call
  with the same counters gives identical results;
* schedules: warp-per-row requantisation (K = 4096, 5120), producer-thread
  requantisation (rows split over warps, K = 25600) and the two-launch path
  for K outside the register schedule;
* grouped launches give exactly the per-matrix nvq_gemv results, with up to
  three matrices per launch (four split into two launches) and M > 1.
"""
import numpy as np
import pytest
import torch

import oracle as o
from bit_weight_quantized_nvq_b200 import capi, workloads as wl
from parity import Packed, assert_within_tolerance, quantize_both, reference

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,K", [(5120, 5120), (25600, 5120), (1024, 4096), (320, 25600),
                                 (640, 1280), (96, 8192)])
def test_requant_is_the_quantiser_of_the_kernels_own_y(N, K):
    W = wl.weights("requant_test", "W", N, K, boost_columns=True)
    x = wl.activations("requant_test", "x", 1, K, "student_t4")
    P = Packed(W)
    q, d, q_ref, d_ref = quantize_both(x)
    counters = torch.zeros(N // 32, dtype=torch.int32, device="cuda")
    y, qo, do = capi.gemv_requant(P.codes, P.scales, P.g, q, d, counters)
    torch.cuda.synchronize()
    y_h = y.cpu().numpy()
    y_ref, sa, _ = reference(P, q_ref, d_ref)
    assert_within_tolerance(y_h, y_ref, sa)
    q_exp, d_exp = o.quantize_q8_0(y_h)
    assert np.array_equal(qo.cpu().numpy(), q_exp), "requantised codes"
    assert np.array_equal(do.cpu().view(torch.int16).numpy().view(np.uint16), d_exp), "scales"
    assert not counters.cpu().numpy().any(), "counters must be left at zero"
    # the plain GEMV writes the same y
    y_plain = capi.gemv(P.codes, P.scales, P.g, q, d)
    torch.cuda.synchronize()
    assert torch.equal(y_plain, y)
    # a second call with the same counters
    y2, qo2, do2 = capi.gemv_requant(P.codes, P.scales, P.g, q, d, counters)
    torch.cuda.synchronize()
    assert torch.equal(y2, y) and torch.equal(qo2, qo) and torch.equal(do2, do)
    assert capi.error_flags() == 0


def test_requant_rejects_ragged_blocks():
    N, K = 48, 256
    codes = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((N, K // 16), dtype=torch.uint8, device="cuda")
    q = torch.zeros((1, K), dtype=torch.int8, device="cuda")
    d = torch.zeros((1, K // 32), dtype=torch.float16, device="cuda")
    counters = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(capi.NVQError) as e:
        capi.gemv_requant(codes, scales, 1.0, q, d, counters, q_out=torch.empty((1, N), dtype=torch.int8, device="cuda"),
                          d_out=torch.empty((1, 2), dtype=torch.float16, device="cuda"))
    assert e.value.status == capi.NVQ_ERR_BAD_SHAPE


@pytest.mark.parametrize("M", [1, 3])
@pytest.mark.parametrize("Ns,K", [((640, 320, 960), 5120), ((2000, 37, 512, 1000), 4096),
                                  ((300, 700), 25600), ((130, 64), 1280)])
def test_grouped_equals_per_matrix(M, Ns, K):
    mats, packed = [], []
    x = wl.activations("group_test", "x", M, K, "student_t4")
    q, d, q_ref, d_ref = quantize_both(x)
    for i, N in enumerate(Ns):
        P = Packed(wl.weights("group_test", f"W{i}", N, K, boost_columns=True))
        packed.append(P)
        mats.append((P.codes, P.scales, P.g))
    ys = capi.gemv_grouped(mats, q, d)
    torch.cuda.synchronize()
    for P, y in zip(packed, ys):
        y_one = capi.gemv(P.codes, P.scales, P.g, q, d)
        torch.cuda.synchronize()
        assert torch.equal(y, y_one)
        y_ref, sa, _ = reference(P, q_ref, d_ref)
        assert_within_tolerance(y.cpu().numpy(), y_ref, sa)
