"""Pins of the oracle's Q8_0 activation quantiser.

Q8_0 holds 32 int8 values and one fp16 scale (34 bytes) per block, per the
GGML type table of the spke.com 2-bit GGUF tutorial (download step).  The
recipe: d32 = amax/127 in fp32, q = rint(x/d32) clamped to +-127, d =
fp16(d32).  The pins are a scalar restatement in plain Python floats (a
double-precision quotient rounded once to fp32 is the correctly rounded fp32
quotient, since 53 >= 2*24 + 2), hand-worked blocks, and invariants.
"""
import struct

import numpy as np
import pytest

import oracle as o
from bit_weight_quantized_nvq_b200 import workloads as wl


def f32(v: float) -> float:
    return struct.unpack("<f", struct.pack("<f", v))[0]


def scalar_q8_0_block(xs):
    """One 32-element block quantised in plain Python scalars."""
    amax = max(abs(v) for v in xs)
    d32 = f32(amax / 127.0)
    if d32 == 0.0:
        q = [0] * len(xs)
    else:
        q = [max(-127, min(127, round(f32(v / d32)))) for v in xs]  # round(): half to even
    d_bits = struct.unpack("<H", struct.pack("<e", d32))[0]
    return q, d_bits


def test_block_geometry_is_32_values_34_bytes():
    x = np.zeros((1, 64), np.float32)
    q, d = o.quantize_q8_0(x)
    assert q.dtype == np.int8 and d.dtype == np.uint16
    assert q.shape == (1, 64) and d.shape == (1, 2)
    assert q[0, :32].nbytes + d[0, :1].nbytes == 34
    with pytest.raises(ValueError):
        o.quantize_q8_0(np.zeros((1, 48), np.float32))


def test_hand_worked_block():
    # amax = 127 -> d32 = 1 exactly, so q = rint(x) with ties to even.
    xs = [127.0, -63.5, 0.5, 1.5, 2.5, -2.5, -0.5, 3.49] + [0.0] * 24
    q, d = o.quantize_q8_0(np.float32([xs]))
    assert list(q[0, :8]) == [127, -64, 0, 2, 2, -2, 0, 3]
    assert list(q[0, 8:]) == [0] * 24
    assert d[0, 0] == 0x3C00              # fp16 1.0
    # amax = 254 -> d32 = 2: 3 -> 1.5 -> 2, 5 -> 2.5 -> 2, -7 -> -3.5 -> -4
    xs = [254.0, 3.0, 5.0, -7.0] + [0.0] * 28
    q, d = o.quantize_q8_0(np.float32([xs]))
    assert list(q[0, :4]) == [127, 2, 2, -4] and d[0, 0] == 0x4000


def test_matches_scalar_restatement_on_random_and_tie_blocks():
    rng = np.random.default_rng(21)
    blocks = [rng.standard_normal(32), rng.standard_t(4, 32) * 10,
              rng.standard_normal(32) * 1e-20, rng.standard_normal(32) * 1e4]
    # exact ties: amax = 127 * 2^k makes d32 = 2^k, and (j + 0.5) * 2^k ties
    for k in (-8, 0, 3):
        b = (rng.integers(-126, 126, 32) + 0.5) * 2.0 ** k
        b[0] = 127 * 2.0 ** k
        blocks.append(b)
    for _ in range(201):
        blocks.append(rng.standard_normal(32) * 2.0 ** rng.uniform(-10, 10))
    x = np.array(blocks, dtype=np.float32).reshape(-1, 64)
    q, d = o.quantize_q8_0(x)
    flat = x.reshape(-1, 32)
    qf = q.reshape(-1, 32)
    df = d.reshape(-1)
    for i, blk in enumerate(flat):
        sq, sd = scalar_q8_0_block([float(v) for v in blk])
        assert list(qf[i]) == sq, i
        assert df[i] == sd, i


def test_invariants_on_workload_activations():
    for x in (wl.activations("small_batch", "x", 16, 5120, "student_t4"),
              wl.activations("prefill", "x", 8, 5120, "normal", outliers=True)):
        q, d = o.quantize_q8_0(x)
        xb = x.reshape(-1, 32).astype(np.float64)
        qb = q.reshape(-1, 32).astype(np.int64)
        assert np.all(np.abs(qb) <= 127)
        amax = np.abs(xb).max(axis=1)
        # the element holding the block's amax quantises to +-127
        arg = np.abs(xb).argmax(axis=1)
        assert np.all(np.abs(qb[np.arange(len(qb)), arg]) == 127)
        # reconstruction with the fp32 d32 is within half a step
        d32 = (amax.astype(np.float32) / np.float32(127)).astype(np.float64)
        err = np.abs(xb - d32[:, None] * qb)
        assert np.all(err <= d32[:, None] * 0.5 * (1 + 2.0 ** -20))
        # the stored fp16 d is within half an fp16 ulp of d32
        dv = o.fp16_values()[d.reshape(-1)]
        assert np.all(np.abs(dv - d32) <= np.abs(d32) * 2.0 ** -11)


def test_zero_block_gives_zero_codes_and_scale():
    x = np.zeros((2, 64), np.float32)
    x[1, 32:] = 1.0
    q, d = o.quantize_q8_0(x)
    assert np.all(q[0] == 0) and np.all(d[0] == 0)
    assert np.all(q[1, :32] == 0) and d[1, 0] == 0
    assert np.all(q[1, 32:] == 127)
