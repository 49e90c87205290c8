"""Kernel timeouts reach the caller.

Every pipeline wait in the kernels is bounded; a wait that runs out raises a
device flag and the kernel returns instead of hanging.  The test makes such a
wait run out on purpose through the test-only nvq_debug_stalled_wait (a
stage whose copy is never issued, limit in microseconds), then reads and
clears the flag through the C ABI, and checks that the context still works:
a GEMV and a GEMM afterwards are correct and raise nothing.  No fault, trap
or endless loop is involved: the wait simply gives up.
"""
import time

import numpy as np
import pytest
import torch

from bit_weight_quantized_nvq_b200 import capi, workloads as wl
from parity import Packed, assert_within_tolerance, quantize_both, reference

pytestmark = pytest.mark.gpu


def test_stalled_wait_returns_and_raises_the_flag():
    torch.cuda.synchronize()
    capi.error_flags(clear=True)
    assert capi.error_flags() == 0
    res = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    limit_us = 300
    t0 = time.time()
    capi.debug_stalled_wait(limit_us * 1000, res)
    torch.cuda.synchronize()
    wall = time.time() - t0
    completed, waited_us = res[:2].cpu().tolist()
    assert completed == 0, "the wait cannot complete"
    assert waited_us >= limit_us, waited_us
    assert wall < 5.0, f"the kernel took {wall:.2f} s to give up"
    flags = capi.error_flags(clear=True)
    assert flags & capi.FLAG_GEMV_TIMEOUT
    assert capi.error_flags() == 0, "clearing the flags did not reset them"


def test_rejects_limits_out_of_range():
    res = torch.zeros((4,), dtype=torch.int32, device="cuda")
    for bad in (0, 10, 2 * 10**9):
        with pytest.raises(capi.NVQError) as e:
            capi.debug_stalled_wait(bad, res)
        assert e.value.status == capi.NVQ_ERR_INVALID_ARG


def test_context_usable_after_a_timeout_and_normal_kernels_raise_nothing():
    res = torch.zeros((4,), dtype=torch.int32, device="cuda")
    capi.debug_stalled_wait(50_000, res)
    torch.cuda.synchronize()
    assert capi.error_flags(clear=True) & capi.FLAG_GEMV_TIMEOUT
    N, K = 300, 5120
    W = wl.weights("errors_test", "W", N, K, boost_columns=True)
    P = Packed(W)
    for M, op in ((1, "gemv"), (4, "gemv"), (200, "gemm")):
        x = wl.activations("errors_test", "x", M, K, "normal")
        q, d, q_ref, d_ref = quantize_both(x)
        if op == "gemv":
            y = capi.gemv(P.codes, P.scales, P.g, q, d)
        else:
            y = capi.gemm(P.codes, P.scales, P.g, q, d)
        torch.cuda.synchronize()
        y_ref, sa, _ = reference(P, q_ref, d_ref)
        assert_within_tolerance(y.cpu().numpy(), y_ref, sa)
    assert capi.error_flags() == 0
    assert np.all(res.cpu().numpy()[:1] == 0)
