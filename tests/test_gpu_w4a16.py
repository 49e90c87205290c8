"""GPU parity of the NVFP4-weight x fp16-activation product (nvq_gemm_w4a16,
the batch-1 decode kernel of "Roofline-First Decoding: results" with NVFP4
weights), against the oracle's dot_fp64_f16:

* shapes the oracle finishes in seconds, every element: one-stage and
  many-stage K, ragged rows, 1..16 tokens, the linear shapes of a
  1.5B-class decoder (hidden 1536, 256-wide key/value, MLP 8960);
* a decode-sweep shape at full size, sampled rows;
* activations near the fp16 maximum, fp16 subnormals and zero tokens;
* fp32 outputs: |y - y_ref| <= 1e-5 * sum_k |w*x| + 1e-6 per element.
"""
import numpy as np
import pytest
import torch

import oracle as o
from bit_weight_quantized_nvq_b200 import capi, workloads as wl
from parity import Packed, assert_within_tolerance, sample_rows, to_dev

pytestmark = pytest.mark.gpu


def fp16_acts(M, K, tag):
    x = wl.activations("w4a16_test", tag, M, K, "student_t4").astype(np.float16)
    x[0, :4] = np.float16(6.0e4)          # near the fp16 maximum
    x[-1, 7] = np.float16(3e-7)           # a subnormal
    return x.view(np.uint16)


@pytest.mark.parametrize("M,N,K", [(1, 37, 256), (1, 1000, 5120), (3, 300, 1536),
                                   (1, 256, 1536), (1, 1536, 8960), (16, 520, 4096),
                                   (9, 129, 2560), (5, 8960, 1536)])
def test_w4a16_all_elements(M, N, K):
    W = wl.weights("w4a16_test", "W", N, K, boost_columns=True)
    P = Packed(W)
    xb = fp16_acts(M, K, "x")
    y = capi.gemm_w4a16(P.codes, P.scales, P.g, to_dev(xb).view(torch.float16))
    torch.cuda.synchronize()
    y_ref = o.dot_fp64_f16(P.ref_codes, P.ref_scales, P.ref_g, xb)
    sa = o.sum_abs_terms_f16(P.ref_codes, P.ref_scales, P.ref_g, xb)
    assert_within_tolerance(y.cpu().numpy(), y_ref, sa)


def test_w4a16_decode_shape_sampled():
    K, N = 5120, 25600
    W, _ = wl.decode_case(K, N)
    rows = sample_rows(N, 256, seed=17)
    P = Packed(W, rows)
    xb = fp16_acts(1, K, "xd")
    y = capi.gemm_w4a16(P.codes, P.scales, P.g, to_dev(xb).view(torch.float16)).cpu().numpy()
    y_ref = o.dot_fp64_f16(P.ref_codes, P.ref_scales, P.ref_g, xb)
    sa = o.sum_abs_terms_f16(P.ref_codes, P.ref_scales, P.ref_g, xb)
    assert_within_tolerance(y[:, rows], y_ref, sa)


def test_zero_token_and_shape_errors():
    M, N, K = 4, 200, 1024
    P = Packed(wl.weights("w4a16_test", "Wz", N, K))
    xb = fp16_acts(M, K, "xz")
    xb[2] = 0
    y = capi.gemm_w4a16(P.codes, P.scales, P.g, to_dev(xb).view(torch.float16)).cpu().numpy()
    assert not y[2].any() and y[0].any()
    bad = torch.zeros((1, 1088), dtype=torch.float16, device="cuda")
    codes = torch.zeros((4, 544), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((4, 68), dtype=torch.uint8, device="cuda")
    with pytest.raises(capi.NVQError) as e:
        capi.gemm_w4a16(codes, scales, 1.0, bad, workspace=torch.empty(1 << 20, dtype=torch.uint8, device="cuda"))
    assert e.value.status == capi.NVQ_ERR_BAD_SHAPE
    assert capi.error_flags() == 0
