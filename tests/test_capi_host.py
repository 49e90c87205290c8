"""Host-side tests of the C ABI: the library loads and exports every symbol
the header declares, host validation returns the documented status codes
before anything is launched, and the host NVFP4 packer is bit-exact against
the oracle's packer.  No GPU is needed."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as o
from bit_weight_quantized_nvq_b200 import capi, workloads as wl

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "nvq.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvq_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 9
    lib = capi.lib()
    for name in names:
        assert hasattr(lib, name), name
        assert name in capi.SIGNATURES, name


def test_version_and_status_strings():
    assert capi.version() >= 10000
    lib = capi.lib()
    for s in range(7):
        assert lib.nvq_status_string(s)
    assert b"unknown" in lib.nvq_status_string(99)
    assert lib.nvq_last_cuda_error() == b"cudaSuccess"


def _dev_like(nbytes, offset=0):
    # host buffers stand in for device pointers: validation never reads them
    buf = np.zeros(nbytes + 64, np.uint8)
    base = buf.ctypes.data
    return buf, (base + (-base % 16) + offset)


def test_host_validation_status_codes():
    lib = capi.lib()
    keep = []
    def p(nbytes=4096, off=0):
        b, a = _dev_like(nbytes, off)
        keep.append(b)
        return a
    codes, scales, q, d, y = p(), p(), p(), p(), p()
    gemv = lib.nvq_gemv
    assert gemv(codes, scales, 1.0, 8, 100, q, d, 1, y, None) == capi.NVQ_ERR_BAD_SHAPE
    assert gemv(codes, scales, 1.0, 8, 0, q, d, 1, y, None) == capi.NVQ_ERR_BAD_SHAPE
    assert gemv(codes, scales, 1.0, 8, 64, q, d, 17, y, None) == capi.NVQ_ERR_BAD_SHAPE
    assert gemv(codes, scales, 1.0, -1, 64, q, d, 1, y, None) == capi.NVQ_ERR_INVALID_ARG
    assert gemv(None, scales, 1.0, 8, 64, q, d, 1, y, None) == capi.NVQ_ERR_INVALID_ARG
    assert gemv(codes, None, 1.0, 8, 64, q, d, 1, y, None) == capi.NVQ_ERR_INVALID_ARG
    assert gemv(codes, scales, 1.0, 8, 64, q, d, 1, p(off=4), None) == capi.NVQ_ERR_MISALIGNED
    assert gemv(p(off=8), scales, 1.0, 8, 64, q, d, 1, y, None) == capi.NVQ_ERR_MISALIGNED
    assert gemv(codes, scales, float("nan"), 8, 64, q, d, 1, y, None) == capi.NVQ_ERR_INVALID_ARG
    # the empty product is a no-op that launches nothing
    assert gemv(codes, scales, 1.0, 0, 64, q, d, 1, y, None) == capi.NVQ_OK
    assert gemv(None, None, 1.0, 8, 64, None, None, 0, None, None) == capi.NVQ_OK

    quant = lib.nvq_quantize_act_q8_0
    assert quant(p(), 1, 48, q, d, None) == capi.NVQ_ERR_BAD_SHAPE
    assert quant(None, 1, 64, q, d, None) == capi.NVQ_ERR_INVALID_ARG
    assert quant(p(off=4), 1, 64, q, d, None) == capi.NVQ_ERR_MISALIGNED
    assert quant(None, 0, 64, None, None, None) == capi.NVQ_OK

    gemm = lib.nvq_gemm
    ws = p(1 << 16)
    need = lib.nvq_gemm_workspace_size(4, 8, 64)
    assert need > 0
    assert gemm(codes, scales, 1.0, 8, 64, q, d, 4, y, None, need, None) == capi.NVQ_ERR_WORKSPACE
    assert gemm(codes, scales, 1.0, 8, 64, q, d, 4, y, ws, need - 1, None) == capi.NVQ_ERR_WORKSPACE
    assert gemm(codes, scales, 1.0, 8, 96, q, d, 4, y, ws, need, None) == capi.NVQ_ERR_BAD_SHAPE
    assert gemm(codes, scales, 1.0, 8, 64, q, d, 4, y, p(1 << 16, 8), need, None) == capi.NVQ_ERR_MISALIGNED
    assert lib.nvq_gemm_workspace_size(0, 8, 64) == 0

    sums = lib.nvq_debug_subblock_sums
    isum = p()
    assert sums(codes, scales, 1.0, 8, 64, q, d, 17, y, isum, None) == capi.NVQ_ERR_BAD_SHAPE
    assert sums(codes, scales, 1.0, 8, 32, q, d, 1, y, isum, None) == capi.NVQ_ERR_BAD_SHAPE
    assert sums(codes, scales, 1.0, 8, 64, q, d, 1, y, None, None) == capi.NVQ_ERR_INVALID_ARG
    assert sums(codes, scales, 1.0, 8, 64, q, d, 1, y, p(off=4), None) == capi.NVQ_ERR_MISALIGNED
    assert sums(None, None, 1.0, 8, 64, None, None, 0, None, None, None) == capi.NVQ_OK

    rq = lib.nvq_gemv_requant
    qo, do, cnt = p(), p(), p()
    assert rq(codes, scales, 1.0, 48, 64, q, d, y, qo, do, cnt, None) == capi.NVQ_ERR_BAD_SHAPE
    assert rq(codes, scales, 1.0, 64, 64, q, d, y, qo, do, None, None) == capi.NVQ_ERR_INVALID_ARG
    assert rq(codes, scales, 1.0, 64, 64, q, d, y, p(off=2), do, cnt, None) == capi.NVQ_ERR_MISALIGNED
    assert rq(codes, scales, 1.0, 64, 96, q, d, y, qo, do, cnt, None) == capi.NVQ_ERR_BAD_SHAPE
    assert rq(codes, scales, 1.0, 0, 64, q, d, y, None, None, None, None) == capi.NVQ_OK

    grouped = lib.nvq_gemv_grouped
    arr = (capi.Linear * 2)(capi.Linear(codes, scales, 1.0, 8, 64),
                            capi.Linear(codes, scales, 1.0, 8, 128))
    ys = (ctypes.c_void_p * 2)(y, y)
    assert grouped(arr, 2, q, d, 1, ys, None) == capi.NVQ_ERR_BAD_SHAPE
    assert grouped(arr, 1, q, d, 17, ys, None) == capi.NVQ_ERR_BAD_SHAPE
    assert grouped(arr, 0, None, None, 1, None, None) == capi.NVQ_OK
    assert grouped(None, 2, q, d, 1, ys, None) == capi.NVQ_ERR_INVALID_ARG

    flags = lib.nvq_error_flags
    assert flags(None, 0) == capi.NVQ_ERR_INVALID_ARG
    stalled = lib.nvq_debug_stalled_wait
    assert stalled(10, p(), None) == capi.NVQ_ERR_INVALID_ARG
    assert stalled(2 * 10**9, p(), None) == capi.NVQ_ERR_INVALID_ARG
    assert stalled(10**6, None, None) == capi.NVQ_ERR_INVALID_ARG
    assert stalled(10**6, p(off=4), None) == capi.NVQ_ERR_MISALIGNED


def test_pack_rejects_bad_arguments():
    lib = capi.lib()
    w = np.zeros((2, 24), np.float32)
    out = np.zeros(64, np.uint8)
    g = ctypes.c_float()
    assert lib.nvq_pack_nvfp4(w.ctypes.data, 2, 24, out.ctypes.data, out.ctypes.data,
                              ctypes.addressof(g)) == capi.NVQ_ERR_BAD_SHAPE
    w = np.zeros((2, 32), np.float32)
    w[1, 3] = np.inf
    assert lib.nvq_pack_nvfp4(w.ctypes.data, 2, 32, out.ctypes.data, out.ctypes.data,
                              ctypes.addressof(g)) == capi.NVQ_ERR_INVALID_ARG
    assert lib.nvq_pack_nvfp4(None, 2, 32, out.ctypes.data, out.ctypes.data,
                              ctypes.addressof(g)) == capi.NVQ_ERR_INVALID_ARG
    with pytest.raises(capi.NVQError):
        capi.pack_nvfp4(np.zeros((2, 40), np.float32))


@pytest.mark.parametrize("case", ["gemv_4096", "decode_boost", "tiny_scales", "zeros",
                                  "ties", "huge_range"])
def test_host_packer_matches_oracle_bit_exactly(case):
    rng = np.random.default_rng(77)
    if case == "gemv_4096":
        w = wl.weights("gemv_4096", "W", 512, 4096)
    elif case == "decode_boost":
        w = wl.weights("decode_sweep", "W", 300, 5120, boost_columns=True)
    elif case == "tiny_scales":
        w = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
        w[:, ::16] *= 1e5                    # one big element per subblock row
        w[3, :] *= 1e-7                      # a row of subnormal-scale subblocks
    elif case == "zeros":
        w = np.zeros((8, 64), np.float32)
    elif case == "ties":
        # exact E2M1 ties: amax 6*448*2^-8 makes g = 2^-8 and s = 1 where the
        # subblock max is 6*2^-8; ratios then land on 0.25, 0.75, ..., 5
        w = np.zeros((4, 64), np.float32)
        base = np.float32(2.0 ** -8)
        w[:, 0] = 6 * 448 * base
        for sb in range(1, 4):
            w[:, sb * 16] = 6 * base
            w[:, sb * 16 + 1:sb * 16 + 8] = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]) * base
            w[1::2, sb * 16 + 1:sb * 16 + 8] *= -1
    else:  # huge_range
        w = (rng.standard_normal((32, 128)) * 10.0 ** rng.uniform(-30, 30, (32, 1))).astype(np.float32)
    c, s, g = capi.pack_nvfp4(w)
    co, so, go = o.pack_nvfp4(w)
    assert np.float32(g) == go
    assert np.array_equal(s, so)
    assert np.array_equal(c, co)


def test_host_validation_of_the_other_entry_points():
    """MoE, W4A16, NVFP4 x NVFP4, the allocation-free GEMM and the decoder
    stack refuse bad arguments on the host, before any device call."""
    lib = capi.lib()
    keep = []

    def p(nbytes=4096, off=0):
        b, a = _dev_like(nbytes, off)
        keep.append(b)
        return a

    codes, scales, q, d, y, ids, gs = p(), p(), p(), p(), p(), p(), p()
    moe = lib.nvq_moe_gemv        # codes, scales, g[E], E, N, K, ids, T, top_k, q, d, y, stream
    assert moe(codes, scales, gs, 4, 64, 96, ids, 2, 2, q, d, y, None) == capi.NVQ_ERR_BAD_SHAPE
    assert moe(codes, scales, gs, 4, 64, 2048, ids, 2, 9, q, d, y, None) == capi.NVQ_ERR_BAD_SHAPE
    assert moe(codes, scales, gs, 0, 64, 2048, ids, 2, 2, q, d, y, None) == capi.NVQ_ERR_INVALID_ARG
    assert moe(codes, scales, gs, 4, 64, 2048, None, 2, 2, q, d, y, None) == capi.NVQ_ERR_INVALID_ARG
    assert moe(codes, scales, gs, 4, 64, 2048, p(off=4), 2, 2, q, d, y, None) == capi.NVQ_ERR_MISALIGNED
    assert moe(codes, scales, gs, 4, 64, 2048, ids, 0, 2, q, d, y, None) == capi.NVQ_OK

    w4 = lib.nvq_gemm_w4a16       # codes, scales, g, N, K, x, M, y, ws, ws_bytes, stream
    assert lib.nvq_gemm_w4a16_workspace_size(17, 8, 256) == 0
    assert lib.nvq_gemm_w4a16_workspace_size(1, 8, 192) == 0
    need = lib.nvq_gemm_w4a16_workspace_size(4, 8, 256)
    assert need > 0
    ws = p(need)
    assert w4(codes, scales, 1.0, 8, 192, q, 4, y, ws, need, None) == capi.NVQ_ERR_BAD_SHAPE
    assert w4(codes, scales, 1.0, 8, 256, q, 17, y, ws, need, None) == capi.NVQ_ERR_BAD_SHAPE
    assert w4(codes, scales, float("nan"), 8, 256, q, 4, y, ws, need, None) == capi.NVQ_ERR_INVALID_ARG
    assert w4(codes, scales, 1.0, 8, 256, q, 4, y, None, need, None) == capi.NVQ_ERR_WORKSPACE
    assert w4(codes, scales, 1.0, 8, 256, q, 4, y, ws, need - 1, None) == capi.NVQ_ERR_WORKSPACE
    assert w4(codes, scales, 1.0, 8, 256, q, 0, y, None, 0, None) == capi.NVQ_OK

    qn = lib.nvq_quantize_act_nvfp4   # x, M, K, codes, scales, g, stream
    assert qn(p(), 2, 24, codes, scales, gs, None) == capi.NVQ_ERR_BAD_SHAPE
    assert qn(None, 2, 32, codes, scales, gs, None) == capi.NVQ_ERR_INVALID_ARG
    assert qn(p(off=4), 2, 32, codes, scales, gs, None) == capi.NVQ_ERR_MISALIGNED
    assert qn(None, 0, 32, None, None, None, None) == capi.NVQ_OK

    nf = lib.nvq_gemm_nvf4        # w_codes, w_scales, g_w, N, K, a_codes, a_scales, a_g, M, y, stream
    assert nf(codes, scales, 1.0, 8, 128, q, d, gs, 4, y, None) == capi.NVQ_ERR_BAD_SHAPE
    assert nf(codes, scales, 1.0, 65535 * 128 + 1, 256, q, d, gs, 4, y, None) == capi.NVQ_ERR_BAD_SHAPE
    assert nf(codes, scales, float("nan"), 8, 256, q, d, gs, 4, y, None) == capi.NVQ_ERR_INVALID_ARG
    assert nf(codes, scales, 1.0, 8, 256, q, d, None, 4, y, None) == capi.NVQ_ERR_INVALID_ARG
    assert nf(codes, scales, 1.0, 8, 256, q, d, gs, 4, p(off=8), None) == capi.NVQ_ERR_MISALIGNED
    assert nf(codes, scales, 1.0, 0, 256, q, d, gs, 4, y, None) == capi.NVQ_OK

    na = lib.nvq_gemm_noalloc     # codes, scales, g, N, K, q, d, M, y, stream
    assert na(codes, scales, 1.0, 8, 96, q, d, 4, y, None) == capi.NVQ_ERR_BAD_SHAPE
    # 2048 tokens of K = 25600 need ~200 MiB of expanded activations
    assert na(codes, scales, 1.0, 128, 25600, q, d, 2048, y, None) == capi.NVQ_ERR_WORKSPACE
    assert na(codes, scales, 1.0, 0, 64, q, d, 4, y, None) == capi.NVQ_OK

    # decoder stack: hidden 64, MLP 128; q k v o up gate down
    shapes = [(64, 64), (64, 64), (64, 64), (64, 64), (128, 64), (128, 64), (64, 128)]

    def layers(n, g=1.0, bad_n=None, off=0):
        arr = (capi.Linear * (7 * n))()
        for l in range(n):
            for i, (N, K) in enumerate(shapes):
                arr[7 * l + i] = capi.Linear(p(off=off), p(), g, N if bad_n != (l, i) else N + 1, K)
        return arr

    outs = (ctypes.c_void_p * 7)(*[p(16384) for _ in range(7)])
    x = p()
    st = lib.nvq_decoder_stack    # linears, n_layers, x, M, outs, ws, ws_bytes, stream
    good = layers(2)
    need = lib.nvq_decoder_stack_workspace_size(good, 1)
    assert need > 0
    ws = p(need)
    assert st(good, 0, x, 1, outs, ws, need, None) == capi.NVQ_OK
    assert st(layers(2, bad_n=(1, 4)), 2, x, 1, outs, ws, need, None) == capi.NVQ_ERR_BAD_SHAPE
    assert st(layers(2, g=float("nan")), 2, x, 1, outs, ws, need, None) == capi.NVQ_ERR_INVALID_ARG
    assert st(layers(2, off=4), 2, x, 1, outs, ws, need, None) == capi.NVQ_ERR_MISALIGNED
    assert st(good, 2, x, 1, outs, ws, need - 1, None) == capi.NVQ_ERR_WORKSPACE
    assert st(good, 2, x, 1, None, ws, need, None) == capi.NVQ_ERR_INVALID_ARG
