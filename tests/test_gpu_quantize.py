"""GPU parity of the fused Q8_0 activation quantiser: codes and fp16 scales
bit-exact against the oracle on the workloads' activations and edge cases."""
import numpy as np
import pytest
import torch

from bit_weight_quantized_nvq_b200 import capi, workloads as wl
from parity import quantize_both, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,dist,outliers", [
    (1, 4096, "normal", False),
    (1, 5120, "normal", False),
    (1, 25600, "normal", False),
    (3, 96, "normal", False),            # ragged: 9 blocks, last warp partial
    (16, 5120, "student_t4", False),
    (7, 25600, "student_t4", False),
    (256, 5120, "normal", True),
    (2048, 5120, "normal", True),        # prefill size, 0.1 % channels x50
    (2048, 25600, "normal", True),
])
def test_workload_activations_bit_exact(M, K, dist, outliers):
    x = wl.activations("quantize_test", "x", M, K, dist, outliers=outliers)
    quantize_both(x)


def test_edge_blocks_bit_exact():
    rng = np.random.default_rng(5)
    x = np.zeros((4, 256), np.float32)
    x[0, 32:64] = 1.0                                    # constant block
    x[0, 64:96] = (np.arange(32) - 16) * 0.5            # exact .5 ties when d32 = 127/127
    x[0, 64] = 127.0
    x[1, :] = rng.standard_normal(256) * 1e-30          # tiny, subnormal d
    x[1, 0:32] = rng.standard_normal(32) * 1e-42        # deep subnormal inputs
    x[2, :] = rng.standard_normal(256) * 3e4            # large d (fp16 range)
    x[3, :] = -np.abs(rng.standard_normal(256))         # all negative
    x[3, 100] = -0.0
    quantize_both(x)


def test_empty_and_no_launch():
    x = torch.zeros((0, 64), device="cuda")
    q, d = capi.quantize_act_q8_0(x)
    assert q.shape == (0, 64) and d.shape == (0, 2)


def test_stream_argument_is_honoured():
    s = torch.cuda.Stream()
    x = wl.activations("quantize_test", "x", 8, 1024, "normal")
    xd = to_dev(x)
    with torch.cuda.stream(s):
        q, d = capi.quantize_act_q8_0(xd, stream=s)
    s.synchronize()
    q2, d2 = capi.quantize_act_q8_0(xd)
    torch.cuda.synchronize()
    assert torch.equal(q, q2) and torch.equal(d, d2)
