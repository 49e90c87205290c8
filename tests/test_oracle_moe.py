"""Pins of the oracle's mixture-of-experts product (mul_mat_id of "HANDOFF:
flint CPU optimization (Q4_1 + NVFP4)", section 7, item 1):

* exact rational brute force on tiny expert sets, decoding with sources
  other than the oracle's own tables;
* each slot equals the single-matrix dot of its expert, computed from the
  dense dequantised expert weights with a plain Python loop;
* permuting a token's slots permutes its outputs; an expert selected twice
  gives two equal outputs; per-expert g scales only that expert's slots;
* ids outside 0..E-1 are refused.
"""
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as o

OCP_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
E4M3 = torch.arange(0, 128, dtype=torch.uint8).view(torch.float8_e4m3fn).double().tolist()


def experts(rng, E, N, K):
    codes = np.empty((E, N, K // 2), np.uint8)
    scales = np.empty((E, N, K // 16), np.uint8)
    g = np.empty(E, np.float32)
    for e in range(E):
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02 * (e + 1))
        codes[e], scales[e], g[e] = o.pack_nvfp4(W)
    return codes, scales, g


def tokens(rng, T, K):
    return o.quantize_q8_0(rng.standard_t(4, size=(T, K)).astype(np.float32))


def test_exact_rational_brute_force():
    rng = np.random.default_rng(1)
    E, N, K, T = 3, 2, 32, 2
    codes, scales, g = experts(rng, E, N, K)
    q, d = tokens(rng, T, K)
    ids = np.array([[2, 0], [1, 2]])
    y = o.moe_dot_fp64(codes, scales, g, ids, q, d)
    for t in range(T):
        for j in range(2):
            e = ids[t, j]
            for n in range(N):
                acc = Fraction(0)
                for k in range(K):
                    byte = int(codes[e, n, k // 2])
                    c = byte & 0xF if k % 2 == 0 else byte >> 4
                    w = Fraction(float(g[e])) * Fraction(E4M3[int(scales[e, n, k // 16])]) \
                        * (-1 if c & 8 else 1) * Fraction(OCP_E2M1[c & 7])
                    a = Fraction(struct.unpack("<e", struct.pack("<H", int(d[t, k // 32])))[0]) * int(q[t, k])
                    acc += w * a
                assert abs(Fraction(y[t, j, n]) - acc) <= abs(acc) * Fraction(1, 2 ** 40) + Fraction(1, 2 ** 100)


def test_slot_equals_dense_loop_of_its_expert():
    rng = np.random.default_rng(2)
    E, N, K, T = 5, 4, 64, 3
    codes, scales, g = experts(rng, E, N, K)
    q, d = tokens(rng, T, K)
    ids = np.array([[4, 1, 3], [0, 0, 2], [1, 4, 2]])
    y = o.moe_dot_fp64(codes, scales, g, ids, q, d)
    a = o.dequantize_activations(q, d)
    for t in range(T):
        for j in range(3):
            w = o.dequantize_weights(codes[ids[t, j]], scales[ids[t, j]], g[ids[t, j]])
            for n in range(N):
                ref = sum(float(w[n, k]) * float(a[t, k]) for k in range(K))
                assert abs(y[t, j, n] - ref) <= 1e-12 * np.abs(w[n] * a[t]).sum()


def test_invariants():
    rng = np.random.default_rng(3)
    E, N, K, T = 6, 8, 128, 2
    codes, scales, g = experts(rng, E, N, K)
    q, d = tokens(rng, T, K)
    ids = np.array([[5, 2, 2, 0], [3, 1, 4, 5]])
    y = o.moe_dot_fp64(codes, scales, g, ids, q, d)
    perm = [2, 0, 3, 1]
    assert np.array_equal(o.moe_dot_fp64(codes, scales, g, ids[:, perm], q, d), y[:, perm])
    assert np.array_equal(y[0, 1], y[0, 2])                   # expert 2 twice
    g2 = g.copy()
    g2[5] *= np.float32(2)
    y2 = o.moe_dot_fp64(codes, scales, g2, ids, q, d)
    assert np.array_equal(y2[0, 0], 2 * y[0, 0]) and np.array_equal(y2[1, 3], 2 * y[1, 3])
    assert np.array_equal(y2[0, 1:], y[0, 1:]) and np.array_equal(y2[1, :3], y[1, :3])
    with pytest.raises(ValueError):
        o.moe_dot_fp64(codes, scales, g, np.array([[6]]), q[:1], d[:1])
