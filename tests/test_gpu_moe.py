"""GPU parity of the mixture-of-experts decode GEMV (nvq_moe_gemv).

* every slot of every token against the oracle's moe_dot_fp64 (all elements)
  on small expert sets, with repeated experts, top_k 1..8, and K on several
  register schedules (K = 2048, 4096, 8192 where rows are split over warps);
* every slot bit-identical to nvq_gemv of its expert (the same kernel code);
* the mixture-of-experts workload shape (256 experts, N = 1536, K = 2048,
  6 of 256 per token) on sampled rows;
* a routing id outside 0..E-1 raises the bad-index flag, leaves its slot
  untouched and does not disturb the other slots;
* fp32 outputs: |y - y_ref| <= 1e-5 * sum|terms| + 1e-6 per element.
"""
import numpy as np
import pytest
import torch

import oracle as o
from bit_weight_quantized_nvq_b200 import capi, workloads as wl
from parity import assert_within_tolerance, quantize_both, to_dev


def pack_experts(E, N, K, tag):
    codes = np.empty((E, N, K // 2), np.uint8)
    scales = np.empty((E, N, K // 16), np.uint8)
    g = np.empty(E, np.float32)
    ref = []
    for e in range(E):
        W = wl.moe_expert_weights(e, N, K, workload=tag)
        codes[e], scales[e], g[e] = capi.pack_nvfp4(W)
        rc, rs, rg = o.pack_nvfp4(W)
        assert np.float32(g[e]) == rg and np.array_equal(codes[e], rc) and np.array_equal(scales[e], rs)
    return codes, scales, g


pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("E,N,K,T,top_k", [(12, 200, 2048, 3, 6), (9, 130, 4096, 2, 8),
                                          (5, 64, 8192, 4, 1), (40, 96, 2048, 16, 6)])
def test_moe_all_slots_against_the_oracle(E, N, K, T, top_k):
    codes, scales, g = pack_experts(E, N, K, f"moe_test_{E}_{K}")
    ids = wl.moe_routing(T, top_k, E, workload=f"moe_test_{E}_{K}")
    ids[0, -1] = ids[0, 0] if top_k > 1 else ids[0, 0]      # an expert chosen twice
    x = wl.activations("moe_test", "x", T, K, "student_t4")
    q, d, q_ref, d_ref = quantize_both(x)
    cd, sd, gd, idd = to_dev(codes), to_dev(scales), to_dev(g), to_dev(ids)
    y = capi.moe_gemv(cd, sd, gd, idd, q, d)
    torch.cuda.synchronize()
    y_ref = o.moe_dot_fp64(codes, scales, g, ids, q_ref, d_ref)
    for t in range(T):
        for j in range(top_k):
            e = ids[t, j]
            isum = o.subblock_sums(codes[e], q_ref[t:t + 1])
            sa = o.sum_abs_terms(isum, scales[e], g[e], d_ref[t:t + 1])
            assert_within_tolerance(y[t, j:j + 1].cpu().numpy(), y_ref[t, j:j + 1], sa)
    # every slot equals nvq_gemv of its expert, bit for bit
    for t in range(T):
        for j in range(top_k):
            e = int(ids[t, j])
            y1 = capi.gemv(cd[e], sd[e], float(g[e]), q[t:t + 1], d[t:t + 1])
            assert torch.equal(y1[0], y[t, j]), (t, j)
    assert capi.error_flags() == 0


def test_moe_workload_shape_sampled_rows():
    E, N, K, top_k, T = wl.MOE_EXPERTS, wl.MOE_N, wl.MOE_K, wl.MOE_TOP_K, 4
    ids = wl.moe_routing(T, top_k, E, step=3)
    used = sorted(set(ids.ravel().tolist()))
    codes = np.zeros((E, N, K // 2), np.uint8)
    scales = np.zeros((E, N, K // 16), np.uint8)
    g = np.zeros(E, np.float32)
    for e in used:                      # only the selected experts are read
        codes[e], scales[e], g[e] = capi.pack_nvfp4(wl.moe_expert_weights(e))
    x = wl.moe_tokens(T)
    q, d, q_ref, d_ref = quantize_both(x)
    y = capi.moe_gemv(to_dev(codes), to_dev(scales), to_dev(g), to_dev(ids), q, d).cpu().numpy()
    rows = np.unique(np.r_[0, N - 1, np.random.default_rng(5).choice(N, 64)])
    for t in range(T):
        for j in range(top_k):
            e = ids[t, j]
            rc, rs, rg = o.pack_nvfp4(wl.moe_expert_weights(e)[rows], g=o.nvfp4_tensor_scale(wl.moe_expert_weights(e)))
            y_ref = o.dot_fp64(rc, rs, rg, q_ref[t:t + 1], d_ref[t:t + 1])
            sa = o.sum_abs_terms(o.subblock_sums(rc, q_ref[t:t + 1]), rs, rg, d_ref[t:t + 1])
            assert_within_tolerance(y[t, j][rows][None, :], y_ref, sa)


def test_bad_routing_id_is_flagged_and_skipped():
    E, N, K, T, top_k = 6, 64, 2048, 2, 3
    codes, scales, g = pack_experts(E, N, K, "moe_test_bad")
    ids = np.array([[1, E, 2], [-1, 0, 5]], np.int32)
    x = wl.activations("moe_test", "xb", T, K, "normal")
    q, d, q_ref, d_ref = quantize_both(x)
    capi.error_flags(clear=True)
    y = torch.full((T, top_k, N), float("nan"), device="cuda")
    capi.moe_gemv(to_dev(codes), to_dev(scales), to_dev(g), to_dev(ids), q, d, y=y)
    torch.cuda.synchronize()
    assert capi.error_flags(clear=True) & capi.FLAG_BAD_INDEX
    yh = y.cpu().numpy()
    assert np.all(np.isnan(yh[0, 1])) and np.all(np.isnan(yh[1, 0]))
    good = np.array([[1, 0, 2], [0, 0, 5]])
    y_ref = o.moe_dot_fp64(codes, scales, g, good, q_ref, d_ref)
    for t, j in ((0, 0), (0, 2), (1, 1), (1, 2)):
        e = good[t, j]
        sa = o.sum_abs_terms(o.subblock_sums(codes[e], q_ref[t:t + 1]), scales[e], g[e], d_ref[t:t + 1])
        assert_within_tolerance(yh[t, j:j + 1], y_ref[t, j:j + 1], sa)


def test_moe_rejects_unsupported_shapes():
    codes = torch.zeros((2, 8, 640 // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((2, 8, 640 // 16), dtype=torch.uint8, device="cuda")
    g = torch.ones(2, device="cuda")
    ids = torch.zeros((1, 2), dtype=torch.int32, device="cuda")
    q = torch.zeros((1, 640), dtype=torch.int8, device="cuda")
    d = torch.zeros((1, 20), dtype=torch.float16, device="cuda")
    with pytest.raises(capi.NVQError) as e:
        capi.moe_gemv(codes, scales, g, ids, q, d)
    assert e.value.status == capi.NVQ_ERR_BAD_SHAPE
