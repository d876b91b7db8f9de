"""Oracle of the block-wise transform with AbsMax-scaled block quantizers (the
WUSH workload: a per-block G x G linear transform of activation rows fused with
activation quantization to MXFP4, NVFP4 or INT4).

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the pages fix (WUSH technical summary, section 2 "method" and
"implementation"): a data-aware linear transform applied per block of G
channels, stored per block (C / G matrices of G x G), fused on the GPU with the
quantization of the activations by a round-to-nearest block quantizer whose scale
comes from the block's absolute maximum, in floating-point (MXFP4, NVFP4) or
integer (INT4) formats.  How the transforms are built (Cholesky factors of the
weight and activation second moments, an SVD, a Hadamard matrix) is offline
work on calibration statistics; here the G x G matrices are inputs.

Readings of what the pages leave open (one quantization group per transform
block, G = 32 for MXFP4 and INT4, G = 16 for NVFP4):

* transform: y[b G + o] = sum_k T[b][o][k] x[b G + k], computed exactly
  (float64 of the bf16 inputs);
* E2M1 (the 4-bit float of MXFP4 and NVFP4): magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}
  with codes 0..7, sign in bit 3; round to nearest, ties to the even code,
  saturating at 6; the sign of a value that rounds to zero is kept (-0 is code 8);
* MXFP4 (OCP microscaling): per group of 32 a shared power-of-two scale
  2^X, X = floor(log2(amax)) - 2 (2 = the largest E2M1 exponent), clamped to
  [-127, 127] and stored as the byte X + 127 (E8M0); X = -127 for an all-zero
  group; elements E2M1(y / 2^X) (exact division by a power of two);
* NVFP4: per group of 16 the scale amax / 6 (float32 division) rounded to FP8
  E4M3 (round to nearest even, saturating at 448, subnormals kept), times a
  per-tensor float32 scale `gscale`; elements E2M1(RN32(y / (s_e4m3 * gscale)))
  with the product and the division in float32; a group whose scale is zero
  codes every element as +0;
* INT4 symmetric AbsMax: per group of 32, scale16 = fp16_RN(RN32(amax / 7)),
  s = float(scale16) (s = 1 when amax == 0 or scale16 underflows to 0),
  q = clamp(rint(RN32(y / s)), -7, 7) (half to even), stored as 4-bit two's
  complement;
* packing: two 4-bit codes per byte, lowest element in the low nibble.
"""

from __future__ import annotations

import numpy as np

E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
FORMATS = {"mxfp4": 32, "nvfp4": 16, "int4": 32}


def block_transform(T, x):
    """y = x transformed block by block: T (C/G, G, G) (float of bf16 values), x (rows, C)."""
    T = np.asarray(T, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    nb, G, G2 = T.shape
    if G != G2 or x.shape[-1] != nb * G:
        raise ValueError("T must be (C/G, G, G) with C the row width")
    xb = x.reshape(x.shape[:-1] + (nb, G))
    y = np.einsum("...bk,bok->...bo", xb, T)
    return y.reshape(x.shape)


def e2m1_code(v):
    """E2M1 codes (uint8, sign in bit 3) of float values: nearest magnitude, ties to the
    even code, saturating at 6; the sign bit follows the sign of v (also for zero)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    # distance to every grid magnitude; ties resolved to the even code index
    d = np.abs(a[..., None] - E2M1_VALUES)
    best = np.argmin(d, axis=-1)
    dmin = np.take_along_axis(d, best[..., None], axis=-1)[..., 0]
    tie = np.sum(d == dmin[..., None], axis=-1) > 1
    # at a tie the two candidates are best and best + 1 (argmin returns the lower):
    # keep the even one
    best = np.where(tie & (best % 2 == 1), best + 1, best)
    best = np.where(a >= 6.0, 7, best)           # saturation (and values above 6)
    sign = np.signbit(v).astype(np.uint8)
    return (sign << 3 | best.astype(np.uint8)).astype(np.uint8)


def e2m1_value(code):
    code = np.asarray(code, dtype=np.uint8)
    mag = E2M1_VALUES[code & 7]
    return np.where(code & 8, -mag, mag)


def e4m3_round(v):
    """Round float values to FP8 E4M3 (finite-only variant): nearest even, saturating at
    448, subnormals (2^-9 steps) kept.  Returns the float64 values."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), 448.0)
    e = np.frexp(np.maximum(a, 2.0 ** -9))[1] - 1.0   # floor(log2 a), exactly
    e = np.maximum(e, -6.0)                      # below 2^-6 the spacing stays 2^-9
    step = 2.0 ** (e - 3)                        # 3 mantissa bits
    q = np.round(a / step) * step                # numpy rounds half to even
    q = np.minimum(q, 448.0)
    return np.where(np.signbit(v), -q, q)


def e4m3_bits(v):
    """FP8 E4M3 bytes (sign, 4 exponent bits biased by 7, 3 mantissa bits) of values that
    are already E4M3-representable (the output of e4m3_round)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    e = np.frexp(np.maximum(a, 2.0 ** -9))[1] - 1
    normal = a >= 2.0 ** -6
    exp_field = np.where(normal, e + 7, 0).astype(np.int64)
    man = np.where(normal, a / 2.0 ** e - 1.0, a / 2.0 ** -6) * 8.0
    bits = (exp_field << 3) | np.rint(man).astype(np.int64)
    bits = np.where(a == 0, 0, bits)
    return (np.signbit(v).astype(np.int64) << 7 | bits).astype(np.uint8)


def _groups(y32, G):
    y32 = np.asarray(y32)
    if y32.dtype != np.float32:
        raise TypeError("the quantizers take float32 input (the values the transform produced)")
    rows, C = y32.shape
    if C % G:
        raise ValueError("group must divide the row width")
    return y32.reshape(rows, C // G, G)


def quantize_mxfp4(y32):
    """(codes (rows, C) uint8, scale bytes (rows, C/32) uint8) of float32 rows."""
    v = _groups(y32, 32).astype(np.float64)
    amax = np.abs(v).max(axis=-1)
    e = np.frexp(np.where(amax > 0, amax, 1.0))[1] - 1        # floor(log2 amax), exactly
    X = np.clip(np.where(amax > 0, e - 2, -127), -127, 127).astype(np.float64)
    q = e2m1_code(v / (2.0 ** X)[..., None])
    return q.reshape(y32.shape), (X + 127).astype(np.uint8)


def quantize_nvfp4(y32, gscale: float = 1.0):
    """(codes (rows, C) uint8, scale (rows, C/16) float32 E4M3 values) of float32 rows
    (the stored scale bytes are e4m3_bits of those values)."""
    v = _groups(y32, 16)
    amax = np.abs(v).max(axis=-1)
    s32 = (amax / np.float32(6.0)).astype(np.float32)
    s8 = e4m3_round(s32).astype(np.float32)
    den = (s8 * np.float32(gscale)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (v / np.where(den == 0, np.float32(1), den)[..., None]).astype(np.float32)
    r = np.where((den == 0)[..., None], np.float32(0.0), r)
    q = e2m1_code(r.astype(np.float64))
    return q.reshape(y32.shape), s8


def quantize_int4_sym(y32):
    """(codes (rows, C) int8 in [-7, 7], scale16 bits (rows, C/32) uint16) of float32 rows."""
    v = _groups(y32, 32)
    amax = np.abs(v).max(axis=-1)
    with np.errstate(over="ignore"):  # beyond the fp16 range the scale rounds to infinity
        s16 = (amax / np.float32(7.0)).astype(np.float32).astype(np.float16)
    s = s16.astype(np.float32)
    bad = (amax == 0) | (s == 0)
    s = np.where(bad, np.float32(1.0), s).astype(np.float32)
    s16 = np.where(bad, np.float16(1.0), s16).astype(np.float16)
    q = np.clip(np.rint(v / s[..., None]), -7, 7).astype(np.int8)
    return q.reshape(y32.shape), s16.view(np.uint16)


def pack4(codes):
    """Two 4-bit codes per byte, lowest element in the low nibble (two's complement nibbles
    for signed input)."""
    c = (np.asarray(codes).astype(np.int16) & 0xF).astype(np.uint8)
    rows, n = c.shape
    c = c.reshape(rows, n // 2, 2)
    return (c[..., 0] | (c[..., 1] << 4)).astype(np.uint8)


def unpack4(packed, signed: bool = False):
    p = np.asarray(packed, dtype=np.uint8)
    lo, hi = p & 0xF, p >> 4
    out = np.stack([lo, hi], axis=-1).reshape(p.shape[0], -1)
    if signed:
        out = np.where(out >= 8, out.astype(np.int16) - 16, out).astype(np.int8)
    return out


def quantize(y32, fmt: str, gscale: float = 1.0):
    """(packed codes (rows, C/2) uint8, scales) of float32 rows in one of the formats; the
    scales are E8M0 bytes (mxfp4), E4M3 bytes (nvfp4) or fp16 bits (int4)."""
    if fmt == "mxfp4":
        q, sc = quantize_mxfp4(y32)
    elif fmt == "nvfp4":
        q, sv = quantize_nvfp4(y32, gscale)
        sc = e4m3_bits(sv)
    elif fmt == "int4":
        q, sc = quantize_int4_sym(y32)
    else:
        raise ValueError(f"unknown format {fmt}")
    return pack4(q), sc


def dequantize(packed, scales, fmt: str, gscale: float = 1.0):
    """float64 values of packed codes (tests only)."""
    if fmt == "int4":
        q = unpack4(packed, signed=True).astype(np.float64)
        s = np.asarray(scales, np.uint16).view(np.float16).astype(np.float64)
        G = 32
    else:
        q = e2m1_value(unpack4(packed))
        G = FORMATS[fmt]
        if fmt == "mxfp4":
            s = 2.0 ** (np.asarray(scales, np.float64) - 127)
        else:
            b = np.asarray(scales, np.uint8).astype(np.int64)
            ex, man = (b >> 3) & 15, b & 7
            mag = np.where(ex > 0, (1.0 + man / 8.0) * 2.0 ** (ex - 7.0), man / 8.0 * 2.0 ** -6)
            s = np.where(b & 128, -mag, mag) * gscale
    rows, n = q.shape
    return (q.reshape(rows, n // G, G) * s[..., None]).reshape(rows, n)
