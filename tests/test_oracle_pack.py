"""Pins of the oracle's NVFP4 weight packer.

Recipe: g = amax/(6*448) in fp32; per 16-element subblock s =
UE4M3(amax_blk/(6g)) and code = nearest E2M1 of w/(g*s), ties to even.  The
pins are a scalar restatement that finds nearest values by brute-force search
over the OCP E2M1 list and PyTorch's E4M3 decoder (not the oracle's grids),
plus round-trip, symmetry and scaling invariants.
"""
import struct

import numpy as np
import torch

import oracle as o
from bit_weight_quantized_nvq_b200 import workloads as wl

OCP_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
E4M3 = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().tolist()


def f32(v: float) -> float:
    return struct.unpack("<f", struct.pack("<f", v))[0]


def nearest_even(v, grid):
    errs = [abs(gv - v) for gv in grid]
    best = min(errs)
    cands = [i for i, e in enumerate(errs) if e == best]
    return cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]


def scalar_pack(w):
    """Plain-Python packer for a small fp32 matrix (list of rows)."""
    amax = max(abs(v) for row in w for v in row)
    g = f32(amax / 2688.0)
    six_g = f32(6.0 * g)
    codes, scales = [], []
    for row in w:
        crow, srow = [], []
        for b in range(0, len(row), 16):
            blk = row[b:b + 16]
            r = f32(max(abs(v) for v in blk) / six_g) if six_g > 0 else 0.0
            s_code = nearest_even(min(r, 448.0), E4M3)
            gs = f32(g * E4M3[s_code])
            for v in blk:
                ratio = f32(v / gs) if gs > 0 else 0.0
                m = nearest_even(min(abs(ratio), 6.0), OCP_E2M1)
                crow.append(m | (8 if (ratio < 0 and m) else 0))
            srow.append(s_code)
        codes.append([crow[i] | (crow[i + 1] << 4) for i in range(0, len(crow), 2)])
        scales.append(srow)
    return np.array(codes, np.uint8), np.array(scales, np.uint8), np.float32(g)


def test_matches_scalar_restatement():
    rng = np.random.default_rng(31)
    for shape, scale in [((3, 64), 0.02), ((2, 128), 1.0), ((4, 64), 1e-3)]:
        w = (rng.standard_normal(shape) * scale).astype(np.float32)
        w[0, 5] *= 20            # a boosted column
        w[1, 16:32] *= 1e-4      # a near-zero subblock (tiny / zero scale)
        c, s, g = o.pack_nvfp4(w)
        sc, ss, sg = scalar_pack([[float(v) for v in row] for row in w])
        assert g == sg
        assert np.array_equal(s, ss)
        assert np.array_equal(c, sc)


def test_nibble_order_low_nibble_is_even_element():
    w = np.zeros((1, 16), np.float32)
    w[0, 0] = 1.0      # the tensor amax: its code is +6 (0x7)
    w[0, 1] = -0.5     # ratio -3 -> code 0xD
    c, s, g = o.pack_nvfp4(w)
    assert c[0, 0] == 0xD7
    assert s[0, 0] == 0x7E and g == np.float32(1.0 / 2688.0)


def test_zero_tensor_packs_to_zeros():
    c, s, g = o.pack_nvfp4(np.zeros((2, 32), np.float32))
    assert g == 0 and not c.any() and not s.any()


def test_round_trip_error_and_block_max_code():
    w = wl.weights("decode_sweep", "W", 64, 5120, boost_columns=True)
    c, s, g = o.pack_nvfp4(w)
    wd = o.dequantize_weights(c, s, g)
    sv = o.UE4M3_VALUES[s]
    step = float(g) * np.repeat(sv, 16, axis=1)          # g*s per element
    ratio = np.abs(w.astype(np.float64)) / np.where(step > 0, step, 1)
    # within half a grid gap of the E2M1 grid (gaps: 0.5 below 2, 1 to 4, 2 to 6),
    # plus the fp32 rounding of w/(g*s), unless saturated beyond 6
    half_gap = np.where(ratio < 2, 0.25, np.where(ratio < 4, 0.5, 1.0))
    err = np.abs(w - wd) / np.where(step > 0, step, 1)
    ok = (err <= half_gap * (1 + 1e-6)) | (ratio > 6)
    assert ok.all()
    # s never exceeds 448, and the element holding a subblock's amax has
    # magnitude code 7 (value 6) whenever the subblock's scale is normal
    assert s.max() <= 0x7E
    codes = o.unpack_codes(c).reshape(64, -1, 16)
    arg = np.abs(w.reshape(64, -1, 16)).argmax(axis=2)
    top = np.take_along_axis(codes, arg[..., None], axis=2)[..., 0] & 7
    normal = s >= 0x08
    assert np.all(top[normal] == 7)


def test_sign_symmetry_and_power_of_two_scaling():
    w = wl.weights("gemv_4096", "W", 16, 256)
    c, s, g = o.pack_nvfp4(w)
    cn, sn, gn = o.pack_nvfp4(-w)
    assert gn == g and np.array_equal(sn, s)
    lo, hi = c & 0xF, c >> 4
    flip = lambda n: np.where(n != 0, n ^ 0x8, 0)
    assert np.array_equal(cn, (flip(lo) | (flip(hi) << 4)).astype(np.uint8))
    c4, s4, g4 = o.pack_nvfp4(w * np.float32(4.0))
    assert g4 == g * 4 and np.array_equal(c4, c) and np.array_equal(s4, s)


def test_subset_rows_with_tensor_scale_match_whole_tensor():
    w = wl.weights("decode_sweep", "W", 40, 512, boost_columns=True)
    c, s, g = o.pack_nvfp4(w)
    rows = np.array([3, 17, 39])
    cr, sr, gr = o.pack_nvfp4(w[rows], g=g)
    assert gr == g and np.array_equal(cr, c[rows]) and np.array_equal(sr, s[rows])
