"""Plain CPU oracle for the NVFP4 x Q8_0 dequantise-and-dot product.

TEST INFRASTRUCTURE, NOT PART OF THE LIBRARY.  Only the test-suite,
``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import this module.  The library never imports it, and it
imports nothing from the library: the two share no code, tables or constants.

What it computes, and the passages it follows
---------------------------------------------
[HANDOFF]  "HANDOFF: flint CPU optimization (Q4_1 + NVFP4)", section 3 "Code
           map (NVFP4 work)": the NVFP4-weight x Q8_0-activation row dot
           (``ggml_vec_dot_nvfp4_q8_0``), weights handled in 64-element blocks
           with one scale per 16 elements (``sd16``), activations as Q8_0
           blocks; and its "Bias trick" paragraph: the integer weight codes
           are stored biased by +12 (0..24), so that
           sum(w*a) = sum((w+12)*a) - 12*bsum16, bsum16 being the sum of the
           16 int8 activation codes of a subblock.
[GGMLTAB]  The spke.com tutorial on 2-bit GGUF builds of a 27B model, the
           GGML type table of its download step: Q8_0 holds 32 values in 34
           bytes (32 int8 codes and one fp16 scale).
[RECIPE]   The NVFP4 / Q8_0 recipe this library is defined by:
           * weights: per-tensor fp32 scale g = amax/(6*448); per 16-element
             subblock a UE4M3 scale s = UE4M3(amax_blk/(6g)); each element an
             E2M1 code, nearest to w/(g*s), ties to even;
           * activations: per 32-element block d32 = amax/127 in fp32,
             q = rint(x/d32) clamped to +-127, stored scale d = fp16(d32);
           * product: per 16-subblock y += g*s_w*d_a*0.5*sum(c_w*q_a) with the
             integer LUT value c_w = 2*E2M1 in -12..12;
           * accuracy: |y - y_ref| <= 1e-5*sum|terms| + 1e-6 per element.
[ROOF]     "Roofline-First Decoding: results": a fused 4-bit dequantise-plus-
           GEMV for batch-1 decoding on fp16 activations (W4A16); here the
           4-bit weights are NVFP4 and the activations binary16 values.
[MOE]      [HANDOFF] section 7 "Open items / next steps", item 1: the NVFP4
           row dot inside a mixture-of-experts product (mul_mat_id: K = 2048,
           256 experts, 6 active per token), each token multiplied by the
           weight matrices of the experts its routing selects.
[NVF4]     NVFP4 on both operands (the Blackwell NVFP4 tensor-core engines
           of "TKintegers K5 ..." and the NVFP4 serving rows of the
           protolabsai lab-benchmarks card): the activations in the weights'
           format, E2M1 codes with one UE4M3 scale per 16, and (reading: the
           pages define NVFP4 only for weights) one fp32 scale per token
           instead of per tensor.
[OCP-MX]   OCP Microscaling Formats (MX) v1.0: the E2M1 element type (1 sign,
           2 exponent bits with bias 1, 1 mantissa bit; max 6) and the E4M3
           type (4 exponent bits with bias 7, 3 mantissa bits, max 448, S.1111.111
           is NaN).  UE4M3 is E4M3 with the sign bit fixed at 0.
[IEEE754]  binary16 (1 sign, 5 exponent bits with bias 15, 10 mantissa bits)
           and round-to-nearest-even.

Readings taken where the passages are silent (each also listed in the design
notes): element 2i of a row sits in the low nibble of byte i and element 2i+1
in the high nibble; codes are stored planar ([N, K/2] code bytes, [N, K/16]
scale bytes); UE4M3 and E2M1 encodes round to nearest, ties to the even code,
and saturate at their largest finite value; an E2M1 result of magnitude zero
is stored as +0; a Q8_0 block whose d32 is 0 quantises to all-zero codes; the
scale arithmetic of the recipe is carried out in fp32 with one IEEE rounding
per operation, left to right as written.

Parity status: every function here is pinned by the tests named in its
docstring (``tests/test_oracle_*.py``).

Floating point: all dot products are evaluated in fp64 (every dequantised
weight and activation is exact in fp64) and the integer subblock sums in
int64.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "e2m1_value", "ue4m3_value", "fp16_value",
    "E2M1_VALUES", "E2M1_INT_LUT", "E2M1_INT_LUT_BIASED", "UE4M3_VALUES",
    "fp16_values",
    "fp32_to_fp16_bits", "fp32_to_ue4m3", "fp32_to_e2m1",
    "quantize_q8_0", "nvfp4_tensor_scale", "pack_nvfp4",
    "unpack_codes", "dequantize_weights", "dequantize_activations",
    "dot_fp64", "subblock_sums", "subblock_sums_biased", "bsum16",
    "y_from_subblock_sums", "sum_abs_terms", "tolerance",
    "dot_fp64_f16", "sum_abs_terms_f16", "moe_dot_fp64",
    "quantize_act_nvfp4", "dot_fp64_nvf4", "sum_abs_terms_nvf4",
    "ACC_REL_TOL", "ACC_ABS_TOL",
]

#: accuracy bound of the fp32 outputs, [RECIPE]
ACC_REL_TOL = 1e-5
ACC_ABS_TOL = 1e-6


# ---------------------------------------------------------------------------
# Format decoders, written from the bit definitions.
# ---------------------------------------------------------------------------

def e2m1_value(code: int) -> float:
    """Real value of a 4-bit E2M1 code [OCP-MX].

    Bit 3 is the sign, bits 2..1 the exponent (bias 1), bit 0 the mantissa.
    Exponent 0 is subnormal: 0.m * 2^0 = m/2.  Otherwise 2^(e-1) * (1 + m/2).
    Pinned by tests/test_oracle_formats.py (the eight OCP magnitudes and the
    0..24 range of the +12-biased integer codes of [HANDOFF] "Bias trick").
    """
    if not 0 <= code <= 15:
        raise ValueError("E2M1 code out of range")
    sign = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        mag = m * 0.5
    else:
        mag = 2.0 ** (e - 1) * (1.0 + m / 2.0)
    return sign * mag


def ue4m3_value(byte: int) -> float:
    """Real value of an unsigned E4M3 scale byte [OCP-MX], NaN for 0x7F.

    Bits 6..3 are the exponent (bias 7), bits 2..0 the mantissa.  Exponent 0
    is subnormal: m/8 * 2^-6.  Bytes with bit 7 set are not UE4M3 values.
    Pinned by tests/test_oracle_formats.py against torch.float8_e4m3fn.
    """
    if not 0 <= byte <= 0x7F:
        raise ValueError("UE4M3 byte out of range (bit 7 must be 0)")
    e = (byte >> 3) & 0xF
    m = byte & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return (m / 8.0) * 2.0 ** -6
    return 2.0 ** (e - 7) * (1.0 + m / 8.0)


def fp16_value(bits: int) -> float:
    """Real value of an IEEE binary16 bit pattern [IEEE754].

    Pinned by tests/test_oracle_formats.py against numpy.float16 over all
    65536 patterns.
    """
    if not 0 <= bits <= 0xFFFF:
        raise ValueError("fp16 bit pattern out of range")
    sign = -1.0 if bits & 0x8000 else 1.0
    e = (bits >> 10) & 0x1F
    m = bits & 0x3FF
    if e == 0x1F:
        return sign * math.inf if m == 0 else math.nan
    if e == 0:
        return sign * (m / 1024.0) * 2.0 ** -14
    return sign * 2.0 ** (e - 15) * (1.0 + m / 1024.0)


#: value of each E2M1 code, fp64 [16]
E2M1_VALUES = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
#: integer LUT c = 2*E2M1 in -12..12 [RECIPE], int64 [16]
E2M1_INT_LUT = np.array([int(2.0 * v) for v in E2M1_VALUES], dtype=np.int64)
#: the same LUT biased by +12, 0..24 [HANDOFF] "Bias trick", int64 [16]
E2M1_INT_LUT_BIASED = E2M1_INT_LUT + 12
#: value of each UE4M3 byte 0x00..0x7F (0x7F is NaN), fp64 [128]
UE4M3_VALUES = np.array([ue4m3_value(b) for b in range(128)], dtype=np.float64)

_FP16_VALUES = None


def fp16_values() -> np.ndarray:
    """Value of every binary16 pattern, fp64 [65536] (built once)."""
    global _FP16_VALUES
    if _FP16_VALUES is None:
        _FP16_VALUES = np.array([fp16_value(b) for b in range(1 << 16)],
                                dtype=np.float64)
    return _FP16_VALUES


# ---------------------------------------------------------------------------
# Encoders: nearest representable value, ties to the even code.
# ---------------------------------------------------------------------------

def _round_nonneg_to_grid(x: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index into ``grid`` of the value nearest to each x (0 <= x <= grid[-1]).

    ``grid`` holds the non-negative values of a format in increasing order,
    indexed by their code, so the lowest code bit is the mantissa's lowest
    bit: a tie between two neighbours goes to the even index.  The midpoint
    of two neighbours is exact in fp64 for every format used here, so every
    comparison is exact.
    """
    x = np.asarray(x, dtype=np.float64)
    lo = np.searchsorted(grid, x, side="right") - 1
    lo = np.clip(lo, 0, len(grid) - 1)
    hi = np.minimum(lo + 1, len(grid) - 1)
    mid = (grid[lo] + grid[hi]) * 0.5
    pick_hi = (x > mid) | ((x == mid) & (hi % 2 == 0) & (hi != lo))
    return np.where(pick_hi, hi, lo)


def fp32_to_fp16_bits(x) -> np.ndarray:
    """binary16 bits of fp32 values, round to nearest even [IEEE754].

    Values of magnitude >= 65520 overflow to infinity.  Pinned against
    numpy's float32 -> float16 conversion (tests/test_oracle_formats.py).
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    finite_pos = fp16_values()[: 0x7C00]          # +0 .. 65504, increasing
    mag = np.abs(x)
    idx = _round_nonneg_to_grid(np.minimum(mag, finite_pos[-1]), finite_pos)
    bits = idx.astype(np.int64)
    bits = np.where(mag >= 65520.0, 0x7C00, bits)
    bits = np.where(np.signbit(x), bits | 0x8000, bits)
    return bits.astype(np.uint16)


def fp32_to_ue4m3(x) -> np.ndarray:
    """UE4M3 byte of non-negative fp32 values: nearest, ties to even, and
    saturating at 448 (0x7E) [OCP-MX]; the reading of "UE4M3(...)" in
    [RECIPE].  Pinned against torch.float8_e4m3fn conversion in range, and by
    brute force nearest-value search (tests/test_oracle_formats.py)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    if np.any(x < 0) or np.any(np.isnan(x)):
        raise ValueError("UE4M3 encodes non-negative finite values only")
    grid = UE4M3_VALUES[:0x7F]                    # 0 .. 448, increasing
    idx = _round_nonneg_to_grid(np.minimum(x, grid[-1]), grid)
    return idx.astype(np.uint8)


def fp32_to_e2m1(x) -> np.ndarray:
    """E2M1 code of fp32 values: nearest magnitude, ties to the even code,
    saturating at 6; a zero magnitude is stored as +0 [OCP-MX], [RECIPE].
    Pinned by brute force nearest search and the tie table
    (tests/test_oracle_formats.py)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    grid = E2M1_VALUES[:8]                        # 0, .5, 1, 1.5, 2, 3, 4, 6
    idx = _round_nonneg_to_grid(np.minimum(np.abs(x), grid[-1]), grid)
    neg = (x < 0) & (idx != 0)
    return (idx | np.where(neg, 0x8, 0)).astype(np.uint8)


# ---------------------------------------------------------------------------
# Q8_0 activation quantiser [GGMLTAB], [RECIPE]
# ---------------------------------------------------------------------------

def quantize_q8_0(x):
    """Q8_0 codes and scales of fp32 activations x [M, K], K % 32 == 0.

    Per 32-element block, in fp32 with one IEEE rounding per operation:
    amax = max|x|, d32 = amax / 127, q = rint(x / d32) (half to even)
    clamped to [-127, 127]; the stored scale is d = fp16(d32) (round to
    nearest even).  A block with d32 == 0 gives q = 0.  Returns
    q int8 [M, K] and d as fp16 bits uint16 [M, K/32].
    Pinned by tests/test_oracle_q8_0.py.
    """
    x = np.asarray(x, dtype=np.float32)
    if x.ndim != 2 or x.shape[1] % 32:
        raise ValueError("x must be [M, K] with K % 32 == 0")
    M, K = x.shape
    xb = x.reshape(M, K // 32, 32)
    amax = np.max(np.abs(xb), axis=2)
    d32 = (amax / np.float32(127.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (xb / d32[:, :, None]).astype(np.float32)
    r = np.where(d32[:, :, None] > 0, r, np.float32(0.0))
    q = np.clip(np.rint(r), -127, 127).astype(np.int8).reshape(M, K)
    d = fp32_to_fp16_bits(d32)
    return q, d


# ---------------------------------------------------------------------------
# NVFP4 weight packer [RECIPE]; layout reading: planar codes and scales.
# ---------------------------------------------------------------------------

def nvfp4_tensor_scale(w) -> np.float32:
    """Per-tensor scale g = amax / (6*448) in fp32 (6*448 = 2688 exactly)."""
    w = np.asarray(w, dtype=np.float32)
    amax = np.float32(np.max(np.abs(w))) if w.size else np.float32(0.0)
    return np.float32(amax / np.float32(2688.0))


def pack_nvfp4(w, g=None):
    """NVFP4 codes, scales and g of fp32 weights w [N, K], K % 16 == 0.

    Per 16-element subblock (fp32, one rounding per operation):
    s = UE4M3(amax_blk / (6*g)); code = E2M1(w / (g*s)).  A subblock whose s
    (or g*s) is 0 stores codes 0.  ``g`` may be given so that a subset of
    rows can be packed with the whole tensor's scale.
    Returns codes uint8 [N, K/2] (element 2i in the low nibble of byte i),
    scales uint8 [N, K/16] and g (np.float32).
    Pinned by tests/test_oracle_pack.py.
    """
    w = np.asarray(w, dtype=np.float32)
    if w.ndim != 2 or w.shape[1] % 16:
        raise ValueError("w must be [N, K] with K % 16 == 0")
    N, K = w.shape
    g = nvfp4_tensor_scale(w) if g is None else np.float32(g)
    wb = w.reshape(N, K // 16, 16)
    amax_blk = np.max(np.abs(wb), axis=2)
    six_g = np.float32(np.float32(6.0) * g)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (amax_blk / six_g).astype(np.float32)
    r = np.where(six_g > 0, r, np.float32(0.0))
    s_code = fp32_to_ue4m3(r)
    s_val = UE4M3_VALUES[s_code].astype(np.float32)
    gs = (g * s_val).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (wb / gs[:, :, None]).astype(np.float32)
    ratio = np.where(gs[:, :, None] > 0, ratio, np.float32(0.0))
    code = fp32_to_e2m1(ratio).reshape(N, K)
    packed = (code[:, 0::2] | (code[:, 1::2] << 4)).astype(np.uint8)
    return packed, s_code.astype(np.uint8), g


# ---------------------------------------------------------------------------
# Dequantise-then-dot in fp64 [HANDOFF] section 3, [RECIPE]
# ---------------------------------------------------------------------------

def unpack_codes(codes) -> np.ndarray:
    """E2M1 code of every element, uint8 [N, K] from code bytes [N, K/2]."""
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty((codes.shape[0], codes.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = codes & 0x0F
    out[:, 1::2] = codes >> 4
    return out


def dequantize_weights(codes, scales, g) -> np.ndarray:
    """w[n, k] = g * UE4M3(scales[n, k//16]) * E2M1(code[n, k]), fp64 [N, K].
    Every product is exact in fp64."""
    c = unpack_codes(codes)
    s = UE4M3_VALUES[np.asarray(scales, dtype=np.uint8)]
    return float(g) * np.repeat(s, 16, axis=1) * E2M1_VALUES[c]


def dequantize_activations(q, d) -> np.ndarray:
    """a[m, k] = fp16(d[m, k//32]) * q[m, k], fp64 [M, K], exact."""
    dv = fp16_values()[np.asarray(d, dtype=np.uint16)]
    return np.repeat(dv, 32, axis=1) * np.asarray(q, dtype=np.float64)


def dot_fp64(codes, scales, g, q, d, row_chunk: int = 4096) -> np.ndarray:
    """y[m, n] = sum_k w[n, k] * a[m, k] in fp64, fp64 [M, N].

    The plain definition: dequantise both operands (exactly) and take their
    dot product; the matrix product is a library primitive.  Rows of W are
    processed in chunks only to bound memory.
    Pinned by exact rational brute force and by agreement with the int64
    path (tests/test_oracle_dot.py).
    """
    a = dequantize_activations(q, d)
    N = np.asarray(codes).shape[0]
    y = np.empty((a.shape[0], N), dtype=np.float64)
    for n0 in range(0, N, row_chunk):
        n1 = min(N, n0 + row_chunk)
        w = dequantize_weights(codes[n0:n1], scales[n0:n1], g)
        y[:, n0:n1] = a @ w.T
    return y


# ---------------------------------------------------------------------------
# Integer subblock path [HANDOFF] "Bias trick", [RECIPE]
# ---------------------------------------------------------------------------

def subblock_sums(codes, q) -> np.ndarray:
    """isum[m, n, sb] = sum over the 16 elements k of subblock sb of
    c_w[n, k] * q[m, k], with c_w = 2*E2M1 in -12..12; int64 [M, N, K/16]."""
    c = E2M1_INT_LUT[unpack_codes(codes)]
    N, K = c.shape
    qq = np.asarray(q, dtype=np.int64)
    M = qq.shape[0]
    return np.einsum("nsj,msj->mns", c.reshape(N, K // 16, 16),
                     qq.reshape(M, K // 16, 16))


def bsum16(q) -> np.ndarray:
    """bsum16[m, sb]: sum of the 16 int8 activation codes of each subblock,
    int64 [M, K/16] [HANDOFF] "Bias trick"."""
    qq = np.asarray(q, dtype=np.int64)
    M, K = qq.shape
    return qq.reshape(M, K // 16, 16).sum(axis=2)


def subblock_sums_biased(codes, q) -> np.ndarray:
    """The same sums through the biased codes of [HANDOFF] "Bias trick":
    sum((c + 12) * q) - 12 * bsum16, int64 [M, N, K/16]."""
    cb = E2M1_INT_LUT_BIASED[unpack_codes(codes)]
    N, K = cb.shape
    qq = np.asarray(q, dtype=np.int64)
    M = qq.shape[0]
    raw = np.einsum("nsj,msj->mns", cb.reshape(N, K // 16, 16),
                    qq.reshape(M, K // 16, 16))
    return raw - 12 * bsum16(q)[:, None, :]


def _subblock_terms(isum, scales, g, d) -> np.ndarray:
    """term[m, n, sb] = 0.5 * g * s_w[n, sb] * d_a[m, sb//2] * isum, fp64."""
    s = UE4M3_VALUES[np.asarray(scales, dtype=np.uint8)]            # [N, S]
    dv = fp16_values()[np.asarray(d, dtype=np.uint16)]              # [M, S/2]
    dv16 = np.repeat(dv, 2, axis=1)                                 # [M, S]
    return (0.5 * float(g)) * s[None, :, :] * dv16[:, None, :] * isum


def y_from_subblock_sums(isum, scales, g, d) -> np.ndarray:
    """y[m, n] = sum_sb 0.5*g*s_w*d_a*isum[m, n, sb] in fp64, [M, N]."""
    return _subblock_terms(isum, scales, g, d).sum(axis=2)


def sum_abs_terms(isum, scales, g, d) -> np.ndarray:
    """sum|terms|[m, n] = sum_sb |0.5*g*s_w*d_a*isum|, fp64 [M, N]: the
    per-element scale of the accuracy bound (reading: the terms are the
    per-subblock contributions)."""
    return np.abs(_subblock_terms(isum, scales, g, d)).sum(axis=2)


def tolerance(sum_abs) -> np.ndarray:
    """Per-element bound 1e-5 * sum|terms| + 1e-6 on |y_fp32 - y_ref|."""
    return ACC_REL_TOL * np.asarray(sum_abs, dtype=np.float64) + ACC_ABS_TOL


# ---------------------------------------------------------------------------
# NVFP4 weights x fp16 activations (W4A16) [ROOF]
# ---------------------------------------------------------------------------

def dot_fp64_f16(codes, scales, g, x_bits, row_chunk: int = 4096) -> np.ndarray:
    """y[m, n] = sum_k w[n, k] * fp16(x_bits[m, k]) in fp64, fp64 [M, N].

    The plain definition for fp16 activations: dequantise the weights and
    decode the binary16 activations (both exact in fp64), then take their
    dot product (a library matrix product).
    Pinned by tests/test_oracle_w4a16.py (exact rational brute force, the
    reduction to dot_fp64 when every activation is a Q8_0 value).
    """
    a = fp16_values()[np.asarray(x_bits, dtype=np.uint16)]
    N = np.asarray(codes).shape[0]
    y = np.empty((a.shape[0], N), dtype=np.float64)
    for n0 in range(0, N, row_chunk):
        n1 = min(N, n0 + row_chunk)
        w = dequantize_weights(codes[n0:n1], scales[n0:n1], g)
        y[:, n0:n1] = a @ w.T
    return y


def sum_abs_terms_f16(codes, scales, g, x_bits, row_chunk: int = 1024) -> np.ndarray:
    """sum|terms|[m, n] = sum_k |w[n, k] * x[m, k]|, fp64 [M, N]: the
    per-element scale of the accuracy bound for fp16 activations.  The
    product has no integer subblock sums, so its terms are the individual
    products w*x (fp32 accumulation of large products that cancel rounds at
    their scale, not at that of their sum)."""
    a = np.abs(fp16_values()[np.asarray(x_bits, dtype=np.uint16)])
    N = np.asarray(codes).shape[0]
    out = np.empty((a.shape[0], N), dtype=np.float64)
    for n0 in range(0, N, row_chunk):
        n1 = min(N, n0 + row_chunk)
        w = np.abs(dequantize_weights(codes[n0:n1], scales[n0:n1], g))
        out[:, n0:n1] = a @ w.T
    return out


# ---------------------------------------------------------------------------
# Mixture-of-experts product (mul_mat_id) [MOE]
# ---------------------------------------------------------------------------

def moe_dot_fp64(codes, scales, g, ids, q, d) -> np.ndarray:
    """y[t, j, n] = sum_k w_{ids[t, j]}[n, k] * a[t, k] in fp64,
    fp64 [T, top_k, N].

    codes [E, N, K/2], scales [E, N, K/16], g [E] (one per-tensor scale per
    expert), ids int [T, top_k] (expert of each slot, every id in 0..E-1),
    q [T, K], d [T, K/32]: each token is multiplied by the matrices of its
    selected experts with the plain dot_fp64.
    Pinned by tests/test_oracle_moe.py.
    """
    codes = np.asarray(codes)
    scales = np.asarray(scales)
    g = np.asarray(g, dtype=np.float32)
    ids = np.asarray(ids)
    T, top_k = ids.shape
    E, N = codes.shape[0], codes.shape[1]
    if np.any(ids < 0) or np.any(ids >= E):
        raise ValueError("expert id out of range")
    y = np.empty((T, top_k, N), dtype=np.float64)
    for t in range(T):
        for j in range(top_k):
            e = int(ids[t, j])
            y[t, j] = dot_fp64(codes[e], scales[e], g[e], q[t:t + 1], d[t:t + 1])[0]
    return y



# ---------------------------------------------------------------------------
# NVFP4 activations, NVFP4 x NVFP4 product [NVF4]
# ---------------------------------------------------------------------------

def quantize_act_nvfp4(x):
    """NVFP4 activations: each token row packed with the weight recipe
    (pack_nvfp4) and its own fp32 scale g[m] = amax(|x[m]|) / (6*448).
    Returns codes uint8 [M, K/2], scales uint8 [M, K/16], g float32 [M].
    Pinned by tests/test_oracle_nvf4.py (and pack_nvfp4's own pins)."""
    x = np.asarray(x, dtype=np.float32)
    M, K = x.shape
    codes = np.empty((M, K // 2), np.uint8)
    scales = np.empty((M, K // 16), np.uint8)
    g = np.empty(M, np.float32)
    for m in range(M):
        codes[m], scales[m], g[m] = pack_nvfp4(x[m:m + 1])
    return codes, scales, g


def dot_fp64_nvf4(w_codes, w_scales, w_g, a_codes, a_scales, a_g) -> np.ndarray:
    """y[m, n] = sum_k w[n, k] * a[m, k] in fp64, fp64 [M, N], with both
    operands NVFP4: w = w_g * UE4M3 * E2M1 (one tensor scale), a[m] = a_g[m] *
    UE4M3 * E2M1 (one scale per token).  Every dequantised value is exact in
    fp64; the matrix product is a library primitive.
    Pinned by tests/test_oracle_nvf4.py."""
    a = np.stack([dequantize_weights(a_codes[m:m + 1], a_scales[m:m + 1], a_g[m])[0]
                  for m in range(np.asarray(a_codes).shape[0])])
    w = dequantize_weights(w_codes, w_scales, w_g)
    return a @ w.T


def sum_abs_terms_nvf4(w_codes, w_scales, w_g, a_codes, a_scales, a_g) -> np.ndarray:
    """sum|terms|[m, n] = sum_k |w[n, k] * a[m, k]|, fp64 [M, N]: the scale
    of the accuracy bound of the NVFP4 x NVFP4 product (its terms are the
    products; there are no integer sums)."""
    a = np.stack([dequantize_weights(a_codes[m:m + 1], a_scales[m:m + 1], a_g[m])[0]
                  for m in range(np.asarray(a_codes).shape[0])])
    w = dequantize_weights(w_codes, w_scales, w_g)
    return np.abs(a) @ np.abs(w).T
