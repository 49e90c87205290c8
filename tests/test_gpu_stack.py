"""GPU parity of the native decoder-stack runner (nvq_decoder_stack).

Each layer restarts from the same input x and chains
Q8_0(x) -> q, k, v;  Q8_0(y_v) -> o;  Q8_0(y_o) -> up, gate;  Q8_0(y_up) -> down,
so the outputs left in the buffers are the last layer's.  The oracle runs the
same chain for that layer in fp64; where a requantised input may sit on the
other side of a rounding tie (the GPU's fp32 input differs from the oracle's
by up to the product tolerance), the next product's bound is widened by the
largest possible change of its dequantised inputs (computed from oracle
values only; zero away from ties).
"""
import numpy as np
import pytest
import torch

import oracle as o
from bit_weight_quantized_nvq_b200 import capi, workloads as wl
from parity import Packed, chained_reference, requant_bound

pytestmark = pytest.mark.gpu

ORDER = ["q", "k", "v", "o", "up", "gate", "down"]


def layer_shapes(h, f):
    return {"q": (h, h), "k": (h, h), "v": (h, h), "o": (h, h),
            "up": (h, f), "gate": (h, f), "down": (f, h)}      # (K, N)


def oracle_chain(packed, x):
    """Per-output (y_ref, tol) of one layer's chain."""
    res = {}
    zero = np.zeros_like(x, dtype=np.float64)
    for name in ("q", "k", "v"):
        res[name] = chained_reference(packed[name], x, zero)
    def requant_input(name):
        y, tol = res[name]
        y32 = y.astype(np.float32)
        # the GPU's fp32 value is within tol of the exact y; the oracle's fp32
        # cast is within half an ulp of it
        t = tol + np.abs(y) * 2.0 ** -24
        return y32, requant_bound(y32, t)
    xv, dv = requant_input("v")
    res["o"] = chained_reference(packed["o"], xv, dv)
    xo, do_ = requant_input("o")
    res["up"] = chained_reference(packed["up"], xo, do_)
    res["gate"] = chained_reference(packed["gate"], xo, do_)
    xu, du = requant_input("up")
    res["down"] = chained_reference(packed["down"], xu, du)
    return res


def build_stack(n_layers, h, f, M, seed_tag):
    shapes = layer_shapes(h, f)
    layers, packed_last = [], None
    for l in range(n_layers):
        layer, packed = [], {}
        for name in ORDER:
            K, N = shapes[name]
            W = wl.weights(f"stack_test/{seed_tag}", f"{name}{l}", N, K)
            P = Packed(W)
            packed[name] = P
            layer.append((P.codes, P.scales, P.g))
        layers.append(layer)
        packed_last = packed
    return capi.DecoderStack(layers, M), packed_last


@pytest.mark.parametrize("M", [1, 3, 16, 40, 130])
def test_small_stack_last_layer_matches_oracle_chain(M):
    h, f = 512, 1024
    stack, packed = build_stack(3, h, f, M, "small")
    x = wl.activations("stack_test", "x", M, h, "normal")
    outs = stack.forward(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    ref = oracle_chain(packed, x)
    for i, name in enumerate(ORDER):
        y = outs[i].cpu().numpy().astype(np.float64)
        y_ref, tol = ref[name]
        err = np.abs(y - y_ref)
        assert np.all(err <= tol), (name, float((err / tol).max()))
        assert np.any(y_ref != 0)


def test_one_token_stack_with_grouped_requantising_launches():
    """One token through shapes that the register schedule covers (K = 4096
    for q/k/v/o/up/gate, 8192 for down): q, k, v in one launch that also
    emits Q8_0(y_v), o emitting Q8_0(y_o), up and gate in one launch emitting
    Q8_0(y_up), down alone; every output of the last layer against the
    oracle chain, and a second pass gives identical outputs (the block
    counters are left at zero)."""
    h, f = 4096, 8192
    stack, packed = build_stack(2, h, f, 1, "grouped")
    x = wl.activations("stack_test", "xg", 1, h, "student_t4")
    xd = torch.from_numpy(x).cuda()
    outs = [t.clone() for t in stack.forward(xd)]
    torch.cuda.synchronize()
    ref = oracle_chain(packed, x)
    for i, name in enumerate(ORDER):
        y = outs[i].cpu().numpy().astype(np.float64)
        y_ref, tol = ref[name]
        err = np.abs(y - y_ref)
        assert np.all(err <= tol), (name, float((err / tol).max()))
        assert np.any(y_ref != 0)
    outs2 = stack.forward(xd)
    torch.cuda.synchronize()
    for a, b in zip(outs, outs2):
        assert torch.equal(a, b)
    assert capi.error_flags() == 0


def per_launch_chain(layer, xd):
    """One layer through the single-matrix entry points (Q8_0 quantiser,
    nvq_gemv, nvq_gemv_requant), the kernels the persistent stack launch
    must reproduce bit for bit."""
    (cq, sq, gq), (ck, sk, gk), (cv, sv, gv), (co, so, go), (cu, su, gu), (cg, sg, gg), \
        (cd, sd, gd) = layer
    cnt = lambda N: torch.zeros(N // 32, dtype=torch.int32, device="cuda")
    qx, dx = capi.quantize_act_q8_0(xd)
    y_q = capi.gemv(cq, sq, gq, qx, dx)
    y_k = capi.gemv(ck, sk, gk, qx, dx)
    y_v, qv, dv = capi.gemv_requant(cv, sv, gv, qx, dx, cnt(cv.shape[0]))
    y_o, qo, do_ = capi.gemv_requant(co, so, go, qv, dv, cnt(co.shape[0]))
    y_u, qu, du = capi.gemv_requant(cu, su, gu, qo, do_, cnt(cu.shape[0]))
    y_g = capi.gemv(cg, sg, gg, qo, do_)
    y_d = capi.gemv(cd, sd, gd, qu, du)
    torch.cuda.synchronize()
    return [y_q, y_k, y_v, y_o, y_u, y_g, y_d]


def test_persistent_one_token_stack_equals_per_launch_kernels():
    """At one token the stack runs as one persistent launch per 64 layers
    (phases separated by grid-wide counters, weights streamed across phase
    boundaries).  Its outputs equal, bit for bit, those of the per-matrix
    launches of the same layer; 66 layers (two launches, the second one
    reusing the phase counters) give the same outputs as one layer, since
    every layer restarts from the same x."""
    h, f = 4096, 8192
    stack1, packed = build_stack(1, h, f, 1, "persistent")
    layer = [(packed[n].codes, packed[n].scales, packed[n].g) for n in ORDER]
    stack66 = capi.DecoderStack([layer] * 66, 1)
    x = wl.activations("stack_test", "xp", 1, h, "student_t4")
    xd = torch.from_numpy(x).cuda()
    ref = per_launch_chain(layer, xd)
    out1 = [t.clone() for t in stack1.forward(xd)]
    out66 = [t.clone() for t in stack66.forward(xd)]
    torch.cuda.synchronize()
    for name, r, a, b in zip(ORDER, ref, out1, out66):
        assert torch.equal(a, r), name
        assert torch.equal(b, r), name
    assert capi.error_flags() == 0


def test_stack_validates_shapes_and_workspace():
    h, f = 256, 512
    stack, _ = build_stack(1, h, f, 2, "val")
    lib = capi.lib()
    arr = stack.linears
    # break the chain: down.K must equal up.N
    bad = (capi.Linear * 7)(*[arr[i] for i in range(7)])
    bad[6].K = 256
    x = torch.zeros((2, h), device="cuda")
    st = lib.nvq_decoder_stack(bad, 1, x.data_ptr(), 2, stack._outs_ptrs,
                               stack.workspace.data_ptr(), stack.workspace.numel(), None)
    assert st == capi.NVQ_ERR_BAD_SHAPE
    st = lib.nvq_decoder_stack(arr, 1, x.data_ptr(), 2, stack._outs_ptrs,
                               stack.workspace.data_ptr(), 16, None)
    assert st == capi.NVQ_ERR_WORKSPACE


@pytest.mark.parametrize("M", [1, 2048])
def test_full_64_layer_stack(M):
    """The 64-layer, 17.9 GB configuration: one layer packed and copied into
    64 device buffers; the last layer's outputs checked against the oracle
    chain (all outputs at M = 1, a token sample at M = 2048)."""
    layer_w = wl.stack_layer_weights()
    packed = {name: Packed(W) for name, W in layer_w}
    host = [(P.codes.cpu(), P.scales.cpu(), P.g) for P in (packed[n] for n in ORDER)]
    layers = [[(c.cuda(), s.cuda(), g) for c, s, g in host] for _ in range(wl.STACK_LAYERS)]
    stack = capi.DecoderStack(layers, M)
    x = wl.stack_input(M)
    outs = stack.forward(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    toks = np.arange(M) if M <= 16 else np.unique(np.r_[0, M - 1, np.random.default_rng(3).choice(M, 6)])
    ref = oracle_chain(packed, x[toks])
    for i, name in enumerate(ORDER):
        y = outs[i].cpu().numpy()[toks].astype(np.float64)
        y_ref, tol = ref[name]
        err = np.abs(y - y_ref)
        assert np.all(err <= tol), (name, float((err / tol).max()))
    del layers, stack
    torch.cuda.empty_cache()
