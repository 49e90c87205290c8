"""Pins of the oracle's dequantise-then-dot (fp64) and integer (int64) paths.

* hand-worked examples (tests/golden/hand_worked_dot.txt);
* exact rational brute force on tiny shapes, decoding with sources other
  than the oracle's own tables (the OCP E2M1 list, PyTorch's E4M3 decoder,
  Python's binary16 unpacking);
* agreement of the fp64 and int64 paths;
* the bias identity sum(c*q) = sum((c+12)*q) - 12*bsum16 of "HANDOFF: flint
  CPU optimization (Q4_1 + NVFP4)", section 3, "Bias trick", on 2^20 blocks;
* invariants: zero scales give zero, flipping the sign of a subblock negates
  its term, doubling g doubles y, permuting rows permutes y;
* planted mistakes in the oracle that these pins must catch.
"""
import os
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as o
import oracle.nvq_oracle as onvq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_dot.txt")
OCP_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
E4M3 = torch.arange(0, 128, dtype=torch.uint8).view(torch.float8_e4m3fn).double().tolist()


def load_golden():
    cases, cur = [], None
    for line in open(GOLDEN):
        t = line.split()
        if not t or t[0].startswith("#"):
            continue
        if t[0] == "case":
            cur = {"name": t[1], "codes": {}, "scales": {}, "q": {}, "d": {},
                   "isum": {}, "y": {}, "sumabs": {}}
        elif t[0] == "shape":
            cur["M"], cur["N"], cur["K"] = map(int, t[1:4])
        elif t[0] == "g":
            cur["g"] = np.float32(float(t[1]))
        elif t[0] in ("codes", "scales"):
            cur[t[0]][int(t[1])] = list(bytes.fromhex(t[2]))
        elif t[0] == "q":
            cur["q"][int(t[1])] = [int(v) for v in t[2:]]
        elif t[0] == "d":
            cur["d"][int(t[1])] = [int(v, 16) for v in t[2:]]
        elif t[0] == "isum":
            cur["isum"][(int(t[1]), int(t[2]))] = [int(v) for v in t[3:]]
        elif t[0] in ("y", "sumabs"):
            cur[t[0]][(int(t[1]), int(t[2]))] = float(t[3])
        elif t[0] == "end":
            M, N, K = cur["M"], cur["N"], cur["K"]
            cur["codes"] = np.array([cur["codes"][n] for n in range(N)], np.uint8)
            cur["scales"] = np.array([cur["scales"][n] for n in range(N)], np.uint8)
            cur["q"] = np.array([cur["q"][m] for m in range(M)], np.int8)
            cur["d"] = np.array([cur["d"][m] for m in range(M)], np.uint16)
            assert cur["codes"].shape == (N, K // 2) and cur["q"].shape == (M, K)
            cases.append(cur)
    return cases


def golden_ok(mod) -> bool:
    """Whether the oracle module reproduces every hand-worked value."""
    for c in load_golden():
        y = mod.dot_fp64(c["codes"], c["scales"], c["g"], c["q"], c["d"])
        isum = mod.subblock_sums(c["codes"], c["q"])
        yi = mod.y_from_subblock_sums(isum, c["scales"], c["g"], c["d"])
        sa = mod.sum_abs_terms(isum, c["scales"], c["g"], c["d"])
        for (m, n), v in c["y"].items():
            if y[m, n] != v or yi[m, n] != v:
                return False
        for (m, n), v in c["sumabs"].items():
            if sa[m, n] != v:
                return False
        for (m, n), v in c["isum"].items():
            if list(isum[m, n]) != v:
                return False
    return True


def brute_force(codes, scales, g, q, d):
    """Exact rational y and integer subblock sums by explicit loops."""
    N, Kh = codes.shape
    K = 2 * Kh
    M = q.shape[0]
    e2m1 = lambda c: (-1 if c & 8 else 1) * OCP_E2M1[c & 7]
    y = [[Fraction(0)] * N for _ in range(M)]
    isum = np.zeros((M, N, K // 16), np.int64)
    for m in range(M):
        dv = [struct.unpack("<e", struct.pack("<H", int(b)))[0] for b in d[m]]
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                byte = int(codes[n, k // 2])
                c = (byte & 0xF) if k % 2 == 0 else (byte >> 4)
                w = Fraction(float(g)) * Fraction(E4M3[int(scales[n, k // 16])]) * Fraction(e2m1(c))
                a = Fraction(dv[k // 32]) * int(q[m, k])
                acc += w * a
                isum[m, n, k // 16] += int(2 * e2m1(c)) * int(q[m, k])
            y[m][n] = acc
    return y, isum


def random_case(rng, M, N, K, scale_lo=0x20, scale_hi=0x60):
    codes = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    scales = rng.integers(scale_lo, scale_hi, (N, K // 16), dtype=np.uint8)
    q = rng.integers(-127, 128, (M, K), dtype=np.int8)
    d = o.fp32_to_fp16_bits(rng.uniform(1e-3, 2.0, (M, K // 32)).astype(np.float32))
    g = np.float32(rng.uniform(1e-5, 1e-3))
    return codes, scales, g, q, d


def test_golden_hand_worked_examples():
    assert golden_ok(onvq)


@pytest.mark.parametrize("M,N,K", [(1, 1, 64), (3, 5, 64), (8, 8, 128), (2, 7, 128)])
def test_exact_rational_brute_force(M, N, K):
    rng = np.random.default_rng(1000 + M * 100 + N * 10 + K)
    codes, scales, g, q, d = random_case(rng, M, N, K)
    y_exact, isum_bf = brute_force(codes, scales, g, q, d)
    y = o.dot_fp64(codes, scales, g, q, d)
    isum = o.subblock_sums(codes, q)
    assert np.array_equal(isum, isum_bf)
    sa = o.sum_abs_terms(isum, scales, g, d)
    for m in range(M):
        for n in range(N):
            assert abs(Fraction(float(y[m, n])) - y_exact[m][n]) <= \
                Fraction(2.0 ** -50) * Fraction(float(sa[m, n]))


def test_exhaustive_single_subblock():
    # every code at every position against every q value: isum = c * q
    codes_all = np.arange(16, dtype=np.uint8)
    for qv in range(-127, 128):
        for c in codes_all:
            codes = np.zeros((1, 8), np.uint8)
            codes[0, 3] = c << 4                 # element 7 (high nibble)
            q = np.zeros((1, 16), np.int8)
            q[0, 7] = qv
            q = np.concatenate([q, np.zeros((1, 16), np.int8)], axis=1)
            codes = np.concatenate([codes, np.zeros((1, 8), np.uint8)], axis=1)
            isum = o.subblock_sums(codes, q)
            sign = -1 if c & 8 else 1
            assert isum[0, 0, 0] == sign * int(2 * OCP_E2M1[c & 7]) * qv


def test_fp64_and_int64_paths_agree_on_workload_shapes():
    from bit_weight_quantized_nvq_b200 import workloads as wl
    W, x = wl.small_batch_case(4, 5120, 25600)
    W = W[:96]
    codes, scales, g = o.pack_nvfp4(W)
    q, d = o.quantize_q8_0(x)
    y = o.dot_fp64(codes, scales, g, q, d)
    isum = o.subblock_sums(codes, q)
    yi = o.y_from_subblock_sums(isum, scales, g, d)
    sa = o.sum_abs_terms(isum, scales, g, d)
    assert np.all(np.abs(y - yi) <= 1e-13 * sa)
    assert np.all(sa > 0) and np.any(y != 0)


def test_bias_identity_on_a_million_blocks():
    rng = np.random.default_rng(41)
    M, N, K = 4, 512, 8192                    # 4*512*512 = 2^20 subblocks
    codes = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    q = rng.integers(-127, 128, (M, K), dtype=np.int8)
    a = o.subblock_sums(codes, q)
    b = o.subblock_sums_biased(codes, q)
    assert a.size == 1 << 20
    assert np.array_equal(a, b)
    assert np.abs(a).max() <= 16 * 12 * 127


def test_invariants():
    rng = np.random.default_rng(42)
    codes, scales, g, q, d = random_case(rng, 3, 6, 256)
    y = o.dot_fp64(codes, scales, g, q, d)
    isum = o.subblock_sums(codes, q)
    # zero scales -> exactly zero
    assert not o.dot_fp64(codes, np.zeros_like(scales), g, q, d).any()
    assert not o.y_from_subblock_sums(isum, np.zeros_like(scales), g, d).any()
    # doubling g doubles y exactly
    assert np.array_equal(o.dot_fp64(codes, scales, np.float32(2 * g), q, d), 2 * y)
    # permuting rows permutes y
    perm = rng.permutation(6)
    # (the integer path exactly; the fp64 path up to the matrix product's
    # own summation order)
    assert np.array_equal(o.subblock_sums(codes[perm], q), isum[:, perm])
    sa = o.sum_abs_terms(isum, scales, g, d)
    yp = o.dot_fp64(codes[perm], scales[perm], g, q, d)
    assert np.all(np.abs(yp - y[:, perm]) <= 1e-14 * sa[:, perm])
    # flipping the sign bit of every code in subblock sb of row n negates
    # that subblock's integer sum and moves y by exactly -2 * its term
    n, sb = 4, 5
    flipped = codes.copy()
    flipped[n, sb * 8:(sb + 1) * 8] ^= 0x88
    isum_f = o.subblock_sums(flipped, q)
    assert np.array_equal(isum_f[:, n, sb], -isum[:, n, sb])
    mask = np.ones_like(isum, bool)
    mask[:, n, sb] = False
    assert np.array_equal(isum_f[mask], isum[mask])
    term = 0.5 * float(g) * o.UE4M3_VALUES[scales[n, sb]] * \
        o.fp16_values()[d[:, sb // 2]] * isum[:, n, sb]
    y_f = o.dot_fp64(flipped, scales, g, q, d)
    assert np.allclose(y_f[:, n] - y[:, n], -2 * term, rtol=0, atol=1e-14)


# --- planted mistakes: each must be caught by the pins above --------------

def _brute_force_ok(mod) -> bool:
    rng = np.random.default_rng(7)
    codes, scales, g, q, d = random_case(rng, 2, 3, 64)
    y_exact, isum_bf = brute_force(codes, scales, g, q, d)
    y = mod.dot_fp64(codes, scales, g, q, d)
    isum = mod.subblock_sums(codes, q)
    if not np.array_equal(isum, isum_bf):
        return False
    return all(abs(float(y_exact[m][n]) - y[m, n]) <= 1e-12 * abs(float(y_exact[m][n])) + 1e-300
               for m in range(2) for n in range(3))


def test_planted_nibble_swap_is_caught(monkeypatch):
    def swapped(codes):
        codes = np.asarray(codes, np.uint8)
        out = np.empty((codes.shape[0], codes.shape[1] * 2), np.uint8)
        out[:, 0::2] = codes >> 4
        out[:, 1::2] = codes & 0xF
        return out
    monkeypatch.setattr(onvq, "unpack_codes", swapped)
    assert not golden_ok(onvq)
    assert not _brute_force_ok(onvq)


def test_planted_wrong_e2m1_entry_is_caught(monkeypatch):
    bad = onvq.E2M1_VALUES.copy()
    bad[6] = 3.5                        # 4.0 mistyped
    monkeypatch.setattr(onvq, "E2M1_VALUES", bad)
    assert not _brute_force_ok(onvq)


def test_planted_scale_index_shift_is_caught(monkeypatch):
    bad = np.concatenate([onvq.UE4M3_VALUES[1:], [np.nan]])   # off by one byte
    monkeypatch.setattr(onvq, "UE4M3_VALUES", bad)
    assert not golden_ok(onvq)
    assert not _brute_force_ok(onvq)


def test_planted_dropped_half_factor_is_caught(monkeypatch):
    real = onvq._subblock_terms
    monkeypatch.setattr(onvq, "_subblock_terms",
                        lambda isum, s, g, d: 2.0 * real(isum, s, g, d))
    assert not golden_ok(onvq)


def test_planted_fp16_bias_error_is_caught(monkeypatch):
    real = onvq.fp16_values()
    monkeypatch.setattr(onvq, "fp16_values", lambda: real * 2.0)
    assert not golden_ok(onvq)
    assert not _brute_force_ok(onvq)


@pytest.mark.parametrize("M,N,K", [(2, 3, 64), (3, 4, 128)])
def test_sum_abs_terms_against_exact_subblock_loop(M, N, K):
    """sum|terms| (the scale of the accuracy bound) against an explicit loop
    over subblocks in exact rationals: |0.5 * g * s_w * d_a * isum| per
    subblock, with isum recomputed from the OCP E2M1 list."""
    rng = np.random.default_rng(7000 + M * 100 + N * 10 + K)
    codes, scales, g, q, d = random_case(rng, M, N, K)
    e2m1 = lambda c: (-1 if c & 8 else 1) * OCP_E2M1[c & 7]
    isum = o.subblock_sums(codes, q)
    sa = o.sum_abs_terms(isum, scales, g, d)
    for m in range(M):
        dv = [struct.unpack("<e", struct.pack("<H", int(b)))[0] for b in d[m]]
        for n in range(N):
            total = Fraction(0)
            for sb in range(K // 16):
                s = 0
                for k in range(16 * sb, 16 * sb + 16):
                    byte = int(codes[n, k // 2])
                    c = (byte & 0xF) if k % 2 == 0 else (byte >> 4)
                    s += int(2 * e2m1(c)) * int(q[m, k])
                term = (Fraction(1, 2) * Fraction(float(g)) * Fraction(E4M3[int(scales[n, sb])])
                        * Fraction(dv[sb // 2]) * s)
                total += abs(term)
            # exact up to the fp64 rounding of the sum (a dropped 0.5 or a
            # wrong scale index would miss by far more)
            assert abs(Fraction(float(sa[m, n])) - total) <= Fraction(2.0 ** -50) * total


def test_tolerance_is_the_stated_bound():
    """|y - y_ref| <= 1e-5 * sum|terms| + 1e-6, elementwise."""
    assert o.tolerance(0.0) == pytest.approx(1e-6, rel=0, abs=1e-18)
    assert o.tolerance(1.0) == pytest.approx(1e-5 + 1e-6, rel=1e-15)
    assert np.allclose(o.tolerance(np.array([2.0, 1e3])), [2e-5 + 1e-6, 1e-2 + 1e-6],
                       rtol=1e-15, atol=0)
