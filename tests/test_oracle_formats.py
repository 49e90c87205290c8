"""Pins of the oracle's format decoders and encoders against outside sources.

Sources: the OCP Microscaling Formats (MX) v1.0 E2M1 value list, PyTorch's
float8_e4m3fn decoder/encoder (UE4M3 is E4M3 with the sign bit 0), numpy's
and Python's own IEEE binary16 conversions, and the 0..24 range of the
+12-biased integer codes stated in "HANDOFF: flint CPU optimization
(Q4_1 + NVFP4)", section 3, "Bias trick".
"""
import struct

import numpy as np
import pytest
import torch

import oracle as o

# OCP MX v1.0, E2M1: the eight non-negative magnitudes in code order.
OCP_E2M1_MAGNITUDES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_values_match_ocp_list():
    assert list(o.E2M1_VALUES[:8]) == OCP_E2M1_MAGNITUDES
    assert list(-o.E2M1_VALUES[8:]) == OCP_E2M1_MAGNITUDES
    # code 0x8 is -0: the sign bit is set and the value is zero
    assert o.E2M1_VALUES[8] == 0.0 and np.signbit(o.E2M1_VALUES[8])


def test_e2m1_integer_lut_and_bias_range():
    # c = 2*E2M1 is an integer in -12..12; biased by +12 it spans 0..24, the
    # range of the unsigned codes in the "Bias trick" paragraph.
    assert list(o.E2M1_INT_LUT[:8]) == [0, 1, 2, 3, 4, 6, 8, 12]
    assert np.all(o.E2M1_INT_LUT[8:] == -o.E2M1_INT_LUT[:8])
    assert o.E2M1_INT_LUT_BIASED.min() == 0 and o.E2M1_INT_LUT_BIASED.max() == 24
    assert np.all(o.E2M1_INT_LUT == 2 * o.E2M1_VALUES)


def test_ue4m3_matches_torch_float8_e4m3fn():
    ref = torch.arange(0, 128, dtype=torch.uint8).view(torch.float8_e4m3fn)
    ref = ref.to(torch.float64).numpy()
    assert np.array_equal(o.UE4M3_VALUES[:127], ref[:127])
    assert np.isnan(o.UE4M3_VALUES[127]) and np.isnan(ref[127])
    assert o.UE4M3_VALUES[0x7E] == 448.0
    assert o.UE4M3_VALUES[0x01] == 2.0 ** -9
    assert o.UE4M3_VALUES[0x38] == 1.0
    with pytest.raises(ValueError):
        o.ue4m3_value(0x80)


def test_fp16_decode_matches_numpy_all_patterns():
    ref = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16).view(np.float16)
    ref = ref.astype(np.float64)
    mine = o.fp16_values()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])
    # sign of zero
    assert np.signbit(mine[0x8000]) and not np.signbit(mine[0])


def _fp16_edge_values():
    h = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = (h[:-1] + h[1:]) / 2            # exact ties between neighbours
    vals = np.concatenate([h, mids, np.nextafter(mids.astype(np.float32), 0),
                           np.nextafter(mids.astype(np.float32), 1e9),
                           [65504.0, 65519.996, 65520.0, 7e4, 1e-9, 2.0 ** -25,
                            2.0 ** -25 * 1.0000001, 3 * 2.0 ** -26]])
    vals = vals.astype(np.float32)
    return np.concatenate([vals, -vals])


def test_fp32_to_fp16_matches_numpy():
    rng = np.random.default_rng(11)
    rand = (rng.uniform(-1, 1, 200_000) *
            2.0 ** rng.uniform(-30, 17, 200_000)).astype(np.float32)
    x = np.concatenate([rand, _fp16_edge_values()])
    mine = o.fp32_to_fp16_bits(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(mine, ref)


def test_fp32_to_fp16_matches_python_struct():
    # Python's struct 'e' packs binary16 with round-half-even (an
    # implementation independent of numpy's).
    rng = np.random.default_rng(12)
    x = (rng.uniform(0, 1, 5000) * 2.0 ** rng.uniform(-26, 15, 5000)).astype(np.float32)
    ref = [struct.unpack("<H", struct.pack("<e", float(v)))[0] for v in x]
    assert list(o.fp32_to_fp16_bits(x)) == ref


def test_fp32_to_ue4m3_matches_torch_in_range():
    grid = o.UE4M3_VALUES[:127]
    mids = (grid[:-1] + grid[1:]) / 2
    rng = np.random.default_rng(13)
    rand = rng.uniform(0, 448, 100_000) * rng.choice([1, 1e-1, 1e-2, 1e-3], 100_000)
    x = np.concatenate([grid, mids, rand]).astype(np.float32)
    x = x[x <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(o.fp32_to_ue4m3(x), ref)


def test_fp32_to_ue4m3_saturates_and_brute_force_nearest():
    assert list(o.fp32_to_ue4m3(np.float32([448, 449, 464, 470, 1e6, 3e38]))) == [0x7E] * 6
    rng = np.random.default_rng(14)
    x = (rng.uniform(0, 1, 3000) * 2.0 ** rng.uniform(-12, 9, 3000)).astype(np.float32)
    x = x[x <= 448]
    codes = o.fp32_to_ue4m3(x)
    vals = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for v, c in zip(x.astype(np.float64), codes):
        err = np.abs(vals - v)
        best = np.flatnonzero(err == err.min())
        assert c in best
        if len(best) == 2:
            assert c % 2 == 0


def test_fp32_to_e2m1_ties_and_saturation():
    # ties go to the even code: 0.25->0, 0.75->1.0, 1.25->1.0, 1.75->2,
    # 2.5->2, 3.5->4, 5->4
    ties = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    expect = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    got = o.E2M1_VALUES[o.fp32_to_e2m1(ties)]
    assert list(got) == expect
    assert list(o.E2M1_VALUES[o.fp32_to_e2m1(-ties)]) == [-v for v in expect]
    # saturation at +-6, zero stored as +0 (code 0)
    assert list(o.fp32_to_e2m1(np.float32([6.5, 100, -7, 0.0, -0.0, -0.2]))) == \
        [0x7, 0x7, 0xF, 0x0, 0x0, 0x0]


def test_fp32_to_e2m1_brute_force_nearest():
    rng = np.random.default_rng(15)
    x = rng.uniform(-7, 7, 20_000).astype(np.float32)
    codes = o.fp32_to_e2m1(x)
    for v, c in zip(x.astype(np.float64), codes):
        mag_code = int(c) & 7
        sign = -1.0 if c & 8 else 1.0
        mags = np.array(OCP_E2M1_MAGNITUDES)
        err = np.abs(mags - min(abs(v), 6.0))
        best = np.flatnonzero(err == err.min())
        assert mag_code in best
        if len(best) == 2:
            assert mag_code % 2 == 0
        if mag_code:
            assert sign == np.sign(v)
        else:
            assert not c & 8
