"""The allocation-free GEMM entry point, nvq_gemm_noalloc.

It serves callers that may not allocate device memory or give the library a
workspace (plugins of frameworks that own every allocation, serving loops
that must not call cudaMalloc): the GEMM's scratch lives in a 64 MiB array
the library keeps on each GPU.  The test calls it through the C ABI, twice
in a row on different problems (the shared scratch keeps the first call's
contents), and checks each result against nvq_gemm with a caller workspace,
within the accuracy bound the other tests use.  This file is collected last
so that a run stopping at the first failure has run everything else first;
it also passes on its own in a fresh process (the first call does the
per-device set-up).
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_weight_quantized_nvq_b200 import capi, workloads as wl
from parity import Packed, assert_within_tolerance, quantize_both, reference

pytestmark = pytest.mark.gpu


def _noalloc(P, q, d, y):
    return capi.lib().nvq_gemm_noalloc(
        P.codes.data_ptr(), P.scales.data_ptr(), ctypes.c_float(P.g), P.N, P.K,
        q.data_ptr(), d.data_ptr(), q.shape[0], y.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


def test_noalloc_gemm_matches_gemm_on_two_calls_in_a_row():
    cases = [(300, 520, 4096), (2048, 640, 5120)]     # (M, N, K); the second fills ~42 MiB
    prepared = []
    for M, N, K in cases:
        W = wl.weights("noalloc_test", "W", N, K, boost_columns=True)
        x = wl.activations("noalloc_test", "x", M, K, "normal", outliers=True)
        P = Packed(W)
        q, d, q_ref, d_ref = quantize_both(x)
        prepared.append((P, q, d, q_ref, d_ref))
    outs = []
    for P, q, d, _, _ in prepared:                     # two calls in a row
        y = torch.full((q.shape[0], P.N), float("nan"), device="cuda")
        assert _noalloc(P, q, d, y) == capi.NVQ_OK
        outs.append(y)
    torch.cuda.synchronize()
    for (P, q, d, q_ref, d_ref), y in zip(prepared, outs):
        y_ws = capi.gemm(P.codes, P.scales, P.g, q, d)
        torch.cuda.synchronize()
        y_ref, sa, _ = reference(P, q_ref, d_ref)
        a, b = y.cpu().numpy(), y_ws.cpu().numpy()
        assert np.all(np.abs(a.astype(np.float64) - b) <= 1e-5 * sa + 1e-6)
        assert_within_tolerance(a, y_ref, sa)


def test_noalloc_gemm_rejects_problems_beyond_its_scratch():
    M, K, N = 2048, 25600, 128                         # needs 200 MiB
    codes = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((N, K // 16), dtype=torch.uint8, device="cuda")
    q = torch.zeros((M, K), dtype=torch.int8, device="cuda")
    d = torch.zeros((M, K // 32), dtype=torch.float16, device="cuda")
    y = torch.zeros((M, N), device="cuda")
    st = capi.lib().nvq_gemm_noalloc(codes.data_ptr(), scales.data_ptr(), ctypes.c_float(1.0),
                                     N, K, q.data_ptr(), d.data_ptr(), M, y.data_ptr(),
                                     torch.cuda.current_stream().cuda_stream)
    assert st == capi.NVQ_ERR_WORKSPACE
