"""Float32-step oracle of per-group asymmetric RTN quantization and INT2/INT4 packing.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages fix only that weights go to 2 bits (explainer article, section
"training & results": W2A16) and that the block quantizer is round-to-nearest
(WUSH technical summary, section 2 "method": RTN block quantizer).  Every step
below is a reading of a silent point, written as explicit float32 operations so
that codes, scales and zero points can be compared bit for bit:

1. groups are ``group`` contiguous elements of a row (group divides n);
   qmax = 2**bits - 1;
2. lo = min(group), hi = max(group) in float32 (the range is NOT widened to
   include zero);
3. scale32 = (hi - lo) / qmax (float32 subtraction, correctly rounded float32
   division); scale16 = fp16 round-to-nearest-even of scale32; quantization
   uses s = float32(scale16) so that dequantizing from the stored values is
   self-consistent;
4. degenerate groups: if hi == lo or s == 0 (fp16 underflow), s = 1.0;
   z = clamp(rint(-lo / s), 0, qmax), an integer stored as fp16 (a zero
   point of 0 is +0.0);  q = clamp(rint(x / s) + z, 0, qmax);
   rint rounds half to even; the divisions are IEEE float32 divisions (never a
   reciprocal multiply);
5. packing is little-endian inside a byte, lowest element index in the lowest
   bits: INT4 byte k = q[2k] | q[2k+1] << 4; INT2 byte k = q[4k] | q[4k+1] << 2
   | q[4k+2] << 4 | q[4k+3] << 6.  codes have shape (rows, n*bits/8); scale and
   zero have shape (rows, n/group) and are fp16 bit patterns (uint16).

Dequantization (tests only): x_hat = (q - z) * s.
"""

from __future__ import annotations

import numpy as np


def _check(n, bits, group):
    if bits not in (2, 4):
        raise ValueError("bits must be 2 or 4")
    if group <= 0 or n % group != 0:
        raise ValueError(f"group {group} must divide the row width {n}")
    if group % (8 // bits) != 0:
        raise ValueError("group must hold a whole number of packed bytes")


def group_params(y32, bits: int, group: int):
    """Per-group (scale16 bits, zero16 bits, s as float32, z as float32) of float32 rows."""
    y32 = np.asarray(y32)
    if y32.dtype != np.float32:
        raise TypeError("the quantizer takes float32 input (the values the transform produced)")
    rows, n = y32.shape
    _check(n, bits, group)
    qmax = np.float32(2 ** bits - 1)
    v = y32.reshape(rows, n // group, group)
    lo = v.min(axis=-1)
    hi = v.max(axis=-1)
    scale32 = (hi - lo) / qmax                       # float32 ops throughout
    scale16 = scale32.astype(np.float16)             # round to nearest even
    s = scale16.astype(np.float32)
    degenerate = (hi == lo) | (s == np.float32(0))
    s = np.where(degenerate, np.float32(1.0), s).astype(np.float32)
    scale16 = np.where(degenerate, np.float16(1.0), scale16).astype(np.float16)
    # the zero point is an integer; +0.0 makes a zero point of 0 encode as +0
    # (rint(-lo/s) of lo = 0 is -0.0, which the clamp may pass through)
    z = (np.clip(np.rint(-lo / s), np.float32(0), qmax) + np.float32(0)).astype(np.float32)
    return scale16.view(np.uint16), z.astype(np.float16).view(np.uint16), s, z


def quantize_codes(y32, bits: int, group: int):
    """Integer codes (rows, n) uint8 plus scale16 / zero16 bit patterns (rows, n/group)."""
    y32 = np.asarray(y32)
    rows, n = y32.shape
    scale16, zero16, s, z = group_params(y32, bits, group)
    qmax = np.float32(2 ** bits - 1)
    v = y32.reshape(rows, n // group, group)
    q = np.rint(v / s[..., None]) + z[..., None]     # float32 division, then rint
    q = np.clip(q, np.float32(0), qmax)
    return q.reshape(rows, n).astype(np.uint8), scale16, zero16


def pack(codes, bits: int):
    """Pack (rows, n) codes into (rows, n*bits/8) bytes, lowest index in the lowest bits."""
    codes = np.asarray(codes, dtype=np.uint8)
    rows, n = codes.shape
    per = 8 // bits
    if n % per:
        raise ValueError("row width must hold a whole number of packed bytes")
    c = codes.reshape(rows, n // per, per).astype(np.uint32)
    out = np.zeros((rows, n // per), dtype=np.uint32)
    for k in range(per):
        out |= c[..., k] << (bits * k)
    return out.astype(np.uint8)


def unpack(packed, bits: int, n: int):
    """Inverse of ``pack``."""
    packed = np.asarray(packed, dtype=np.uint8)
    rows = packed.shape[0]
    per = 8 // bits
    mask = (1 << bits) - 1
    c = np.empty((rows, packed.shape[1], per), dtype=np.uint8)
    for k in range(per):
        c[..., k] = (packed >> (bits * k)) & mask
    return c.reshape(rows, n)


def quantize_pack(y32, bits: int, group: int):
    """(packed codes, scale16 bits, zero16 bits) of float32 rows: the fused epilogue's output."""
    codes, scale16, zero16 = quantize_codes(y32, bits, group)
    return pack(codes, bits), scale16, zero16


def dequantize(codes, scale16, zero16, group: int):
    """x_hat = (q - z) * s in float32 from unpacked codes and fp16 bit patterns."""
    codes = np.asarray(codes)
    rows, n = codes.shape
    s = np.asarray(scale16, dtype=np.uint16).view(np.float16).astype(np.float32)
    z = np.asarray(zero16, dtype=np.uint16).view(np.float16).astype(np.float32)
    q = codes.reshape(rows, n // group, group).astype(np.float32)
    return ((q - z[..., None]) * s[..., None]).reshape(rows, n)
