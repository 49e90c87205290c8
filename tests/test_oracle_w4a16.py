"""Pins of the oracle's NVFP4-weight x fp16-activation dot (W4A16, the
batch-1 decode kernel of "Roofline-First Decoding: results" with NVFP4
weights):

* exact rational brute force on tiny shapes, decoding with sources other
  than the oracle's own tables (the OCP E2M1 list, PyTorch's E4M3 decoder,
  Python's binary16 unpacking);
* reduction to the Q8_0 path: when every activation is an exact Q8_0 value
  d*q, the fp16 dot equals dot_fp64 on (q, d) exactly;
* the accuracy-bound scale (sum of |w*x| over k) against an exact loop, and
  its relation to the Q8_0 path's per-subblock scale;
* invariants: zero activations and zero scales give zero, negating the
  activations negates y, x2 on g doubles y;
* a planted mistake (activation decoded with a wrong exponent bias) is
  caught.
"""
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as o
import oracle.nvq_oracle as onvq

OCP_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
E4M3 = torch.arange(0, 128, dtype=torch.uint8).view(torch.float8_e4m3fn).double().tolist()


def fp16_bits(x):
    return np.asarray(x, dtype=np.float16).view(np.uint16)


def e2m1_exact(c):
    v = Fraction(OCP_E2M1[c & 7]).limit_denominator(4)
    return -v if c & 8 else v


def half_exact(bits):
    return Fraction(struct.unpack("<e", struct.pack("<H", int(bits)))[0])


def random_case(rng, M, N, K):
    W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
    W[:, rng.choice(K, 2, replace=False)] *= np.float32(20)
    codes, scales, g = o.pack_nvfp4(W)
    x = rng.standard_t(4, size=(M, K)).astype(np.float16)
    x[:, :3] = np.float16(6e4) * np.sign(x[:, :3])        # near the fp16 maximum
    x[0, 5] = np.float16(3e-7)                             # a subnormal
    return codes, scales, g, x.view(np.uint16)


@pytest.mark.parametrize("M,N,K", [(1, 3, 16), (2, 4, 32), (3, 2, 64)])
def test_exact_rational_brute_force(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    codes, scales, g, xb = random_case(rng, M, N, K)
    y = o.dot_fp64_f16(codes, scales, g, xb)
    gf = Fraction(float(g))
    for m in range(M):
        for n in range(N):
            acc, mag = Fraction(0), Fraction(0)
            for k in range(K):
                byte = int(codes[n, k // 2])
                c = byte & 0xF if k % 2 == 0 else byte >> 4
                w = gf * Fraction(E4M3[int(scales[n, k // 16])]) * e2m1_exact(c)
                acc += w * half_exact(xb[m, k])
                mag += abs(w * half_exact(xb[m, k]))
            # every product is exact in fp64; the sum rounds at most K times
            assert abs(Fraction(y[m, n]) - acc) <= mag * K * Fraction(1, 2 ** 53)


def test_reduces_to_the_q8_0_dot_on_q8_0_values():
    rng = np.random.default_rng(7)
    M, N, K = 3, 40, 256
    W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
    codes, scales, g = o.pack_nvfp4(W)
    q = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    # power-of-two d: d*q is an exact binary16 value
    d_vals = (2.0 ** rng.integers(-12, -2, size=(M, K // 32))).astype(np.float16)
    d = d_vals.view(np.uint16)
    x = (np.repeat(d_vals.astype(np.float64), 32, axis=1) * q).astype(np.float16)
    assert np.array_equal(x.astype(np.float64),
                          np.repeat(d_vals.astype(np.float64), 32, axis=1) * q)
    y16 = o.dot_fp64_f16(codes, scales, g, x.view(np.uint16))
    y8 = o.dot_fp64(codes, scales, g, q, d)
    assert np.allclose(y16, y8, rtol=1e-15, atol=0)
    # the per-element terms bound the Q8_0 path's per-subblock terms
    isum = o.subblock_sums(codes, q)
    sa16 = o.sum_abs_terms_f16(codes, scales, g, x.view(np.uint16))
    assert np.all(sa16 >= o.sum_abs_terms(isum, scales, g, d) * (1 - 1e-15))


def test_sum_abs_terms_against_exact_loop():
    rng = np.random.default_rng(11)
    M, N, K = 2, 3, 64
    codes, scales, g, xb = random_case(rng, M, N, K)
    got = o.sum_abs_terms_f16(codes, scales, g, xb)
    gf = Fraction(float(g))
    for m in range(M):
        for n in range(N):
            tot = Fraction(0)
            for k in range(K):
                byte = int(codes[n, k // 2])
                c = byte & 0xF if k % 2 == 0 else byte >> 4
                tot += abs(gf * Fraction(E4M3[int(scales[n, k // 16])]) * e2m1_exact(c) * half_exact(xb[m, k]))
            # a sum of non-negative fp64 values rounds by at most K ulps
            assert abs(Fraction(got[m, n]) - tot) <= tot * K * Fraction(1, 2 ** 53)


def test_invariants():
    rng = np.random.default_rng(5)
    codes, scales, g, xb = random_case(rng, 2, 20, 128)
    y = o.dot_fp64_f16(codes, scales, g, xb)
    assert np.any(y != 0)
    assert not o.dot_fp64_f16(codes, scales, g, np.zeros_like(xb)).any()
    assert not o.dot_fp64_f16(codes, np.zeros_like(scales), g, xb).any()
    assert np.array_equal(o.dot_fp64_f16(codes, scales, g, xb ^ np.uint16(0x8000)), -y)
    assert np.array_equal(o.dot_fp64_f16(codes, scales, np.float32(2) * g, xb), 2 * y)


def test_planted_activation_decode_error_is_caught(monkeypatch):
    rng = np.random.default_rng(3)
    codes, scales, g, xb = random_case(rng, 1, 2, 32)
    good = o.dot_fp64_f16(codes, scales, g, xb)
    wrong = o.fp16_values() * 2.0                 # exponent bias off by one
    monkeypatch.setattr(onvq, "fp16_values", lambda: wrong)
    bad = onvq.dot_fp64_f16(codes, scales, g, xb)
    assert not np.allclose(bad, good)
