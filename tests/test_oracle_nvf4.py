"""Pins of the oracle's NVFP4-activation quantiser and NVFP4 x NVFP4 dot:

* the quantiser packs every token with its own tensor scale amax/2688 and
  is the weight packer on that row (whose own pins cover the rounding);
* exact rational brute force of the dot with independent decoders (the OCP
  E2M1 list, PyTorch's E4M3 decoder);
* the bound scale against an exact loop;
* invariants: swapping the roles of the operands transposes y; x2 on a
  token's scale doubles its row; zero scales give zero.
"""
from fractions import Fraction

import numpy as np
import torch

import oracle as o

OCP_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
E4M3 = torch.arange(0, 128, dtype=torch.uint8).view(torch.float8_e4m3fn).double().tolist()


def exact(codes, scales, g, r, k):
    byte = int(codes[r, k // 2])
    c = byte & 0xF if k % 2 == 0 else byte >> 4
    v = Fraction(OCP_E2M1[c & 7])
    return Fraction(float(g)) * Fraction(E4M3[int(scales[r, k // 16])]) * (-v if c & 8 else v)


def case(rng, M, N, K):
    W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
    wc, ws, wg = o.pack_nvfp4(W)
    x = rng.standard_t(4, size=(M, K)).astype(np.float32)
    x[0] *= np.float32(300)                       # tokens of very different size
    ac, as_, ag = o.quantize_act_nvfp4(x)
    return x, (wc, ws, wg), (ac, as_, ag)


def test_quantiser_is_the_packer_per_token():
    rng = np.random.default_rng(1)
    x, _, (ac, as_, ag) = case(rng, 5, 4, 64)
    for m in range(5):
        assert ag[m] == np.float32(np.float32(np.abs(x[m]).max()) / np.float32(2688.0))
        c, s, g = o.pack_nvfp4(x[m:m + 1])
        assert np.array_equal(c[0], ac[m]) and np.array_equal(s[0], as_[m]) and g == ag[m]


def test_exact_rational_brute_force():
    rng = np.random.default_rng(2)
    M, N, K = 3, 2, 48
    _, (wc, ws, wg), (ac, as_, ag) = case(rng, M, N, K)
    y = o.dot_fp64_nvf4(wc, ws, wg, ac, as_, ag)
    sa = o.sum_abs_terms_nvf4(wc, ws, wg, ac, as_, ag)
    for m in range(M):
        for n in range(N):
            acc, mag = Fraction(0), Fraction(0)
            for k in range(K):
                t = exact(wc, ws, wg, n, k) * exact(ac, as_, ag[m], m, k)
                acc += t
                mag += abs(t)
            assert abs(Fraction(y[m, n]) - acc) <= mag * K * Fraction(1, 2 ** 53)
            assert abs(Fraction(sa[m, n]) - mag) <= mag * K * Fraction(1, 2 ** 53)


def test_invariants():
    rng = np.random.default_rng(3)
    _, (wc, ws, wg), (ac, as_, ag) = case(rng, 4, 6, 128)
    y = o.dot_fp64_nvf4(wc, ws, wg, ac, as_, ag)
    assert np.any(y != 0)
    yt = o.dot_fp64_nvf4(ac, as_, np.float32(1), wc, ws, np.full(6, wg, np.float32))
    assert np.allclose(yt.T * ag[:, None], y, rtol=1e-14, atol=0)
    ag2 = ag.copy()
    ag2[2] *= np.float32(2)
    y2 = o.dot_fp64_nvf4(wc, ws, wg, ac, as_, ag2)
    assert np.array_equal(y2[2], 2 * y[2]) and np.array_equal(np.delete(y2, 2, 0), np.delete(y, 2, 0))
    assert not o.dot_fp64_nvf4(wc, np.zeros_like(ws), wg, ac, as_, ag).any()
