"""Shared helpers of the GPU parity tests: device transfers and the comparison rules.

Comparison rules (per the accuracy bounds of the transform path):
* float32 outputs: per row, max |y_gpu - y_oracle| <= 2e-5 * ||x||_2;
* bfloat16 outputs: bitwise the round-to-nearest-even of the GPU's own float32
  output, and within one bf16 ulp of the oracle plus the float32 bound (a
  literal one-ulp bound is unreachable for elements much smaller than 2e-5 ||x||);
* quantized codes, scales and zero points computed from identical float32
  inputs are bit-exact; end to end, codes may differ by one level in at most
  1e-4 of the entries, and only at rounding ties: every differing code must sit
  next to a decision boundary of the oracle's quantizer, within the GPU's own
  transform error of that element (plus the boundary's shift when the group's
  scale or zero point came out different);
* dtheta: |gpu - oracle| <= 2e-4 * A + 1e-6 * max(A), A = sum of |terms|.
"""

from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from rotation_bit_quantization_b200 import workloads as wl

F32_TOL = 2e-5


def torch():
    import torch as t
    return t


def dev_f32(a):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def dev_bf16_bits(bits):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).cuda().view(t.bfloat16)


def host(t_):
    t = torch()
    if t_.dtype == t.bfloat16:
        return t_.view(t.int16).cpu().numpy().view(np.uint16)
    return t_.cpu().numpy()


def input_f64(w_x, dtype):
    return (wl.f32_from_bf16_bits(w_x) if dtype == "bf16" else np.asarray(w_x, np.float32)).astype(np.float64)


def assert_f32_close(y_gpu, y_ref, x_ref, tol=F32_TOL):
    y_gpu = np.asarray(y_gpu, np.float64).reshape(y_ref.shape)
    err = np.abs(y_gpu - y_ref).max(axis=-1)
    bound = tol * np.linalg.norm(x_ref, axis=-1)
    worst = int(np.argmax(err - bound))
    assert np.all(err <= bound), f"row {worst}: err {err[worst]:.3e} > bound {bound[worst]:.3e}"
    return float((err / np.maximum(np.linalg.norm(x_ref, axis=-1), 1e-300)).max())


def _ordered(bits):
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def bf16_ulp(v):
    v = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_bf16_output(bits_gpu, y32_gpu, y_ref, x_ref, tol=F32_TOL):
    """bf16 output = RN(GPU float32 output) bitwise; |bf16 - oracle| <= ulp(oracle) + tol * ||x||."""
    bits_gpu = np.asarray(bits_gpu, np.uint16).reshape(y_ref.shape)
    assert np.array_equal(bits_gpu, wl.bf16_bits_from_f32(np.asarray(y32_gpu, np.float32).reshape(y_ref.shape))), \
        "bf16 output is not the rounding of the float32 output"
    v = wl.f32_from_bf16_bits(bits_gpu).astype(np.float64)
    bound = bf16_ulp(y_ref) + tol * np.linalg.norm(x_ref, axis=-1, keepdims=True)
    err = np.abs(v - y_ref)
    assert np.all(err <= bound), f"bf16 error {err.max():.3e} above bound"
    ref_bits = wl.bf16_bits_from_f32(np.asarray(y_ref, np.float64).astype(np.float32))
    return float((np.abs(_ordered(bits_gpu) - _ordered(ref_bits)) > 1).mean())


def ordered_diff_codes(a, b):
    return np.abs(a.astype(np.int32) - b.astype(np.int32))


def oracle_rows(fn, x, chunk: int = 64):
    """fn applied to row chunks of x on a thread pool (numpy releases the GIL), rows in order.

    Used to run the float64 oracle over every row of the full workloads in seconds."""
    x = np.asarray(x)
    starts = list(range(0, x.shape[0], chunk))
    workers = max(1, min(len(starts), len(os.sched_getaffinity(0))))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        parts = list(ex.map(lambda s: fn(x[s:s + chunk]), starts))
    return np.concatenate(parts, axis=0)


def assert_codes_tie_local(q_gpu, s16_gpu, z16_gpu, y_gpu, q_ref, s16_ref, z16_ref, y_ref32, group):
    """End-to-end code agreement: every differing code is one level off and explained by a rounding tie.

    q_* are unpacked codes (rows, n); s16/z16 fp16 bit patterns (rows, n/group); y_gpu the
    kernel's float32 output and y_ref32 the oracle's float64 transform rounded to float32 (the
    values each side quantized).  A code q differs from q + 1 at the decision boundary
    B = (q + 1/2 - z) * s.  Codes are monotone in y, so a mismatch between levels q and q + 1
    is a tie only if the oracle's value lies within |y_gpu - y_ref| (the transform error of
    that very element) of the oracle's boundary, widened by how far the GPU's boundary moved
    when its group's scale or zero point differ, and by a few float32 ulps (the quantizer's
    division rounds once).  Returns (mismatch fraction, largest boundary distance in units
    of the allowed distance)."""
    q_gpu = np.asarray(q_gpu, np.int32)
    q_ref = np.asarray(q_ref, np.int32)
    d = np.abs(q_gpu - q_ref)
    assert d.max(initial=0) <= 1, f"codes differ by {d.max()} levels"
    frac = float((d > 0).mean())
    assert frac <= 1e-4, f"end-to-end code mismatch on {frac:.2e} of the entries (> 1e-4)"
    r, c = np.nonzero(d)
    if r.size == 0:
        return frac, 0.0
    g = c // group

    def sz(s16, z16):
        s = np.asarray(s16, np.uint16).view(np.float16).astype(np.float64)[r, g]
        z = np.asarray(z16, np.uint16).view(np.float16).astype(np.float64)[r, g]
        return s, z

    s_g, z_g = sz(s16_gpu, z16_gpu)
    s_r, z_r = sz(s16_ref, z16_ref)
    q_lo = np.minimum(q_gpu[r, c], q_ref[r, c]).astype(np.float64)
    b_r = (q_lo + 0.5 - z_r) * s_r
    b_g = (q_lo + 0.5 - z_g) * s_g
    yr = np.asarray(y_ref32, np.float64)[r, c]
    yg = np.asarray(y_gpu, np.float64)[r, c]
    allowed = np.abs(yg - yr) + np.abs(b_g - b_r) + 4.0 * np.spacing(np.abs(b_r).astype(np.float32)).astype(np.float64)
    dist = np.abs(yr - b_r)
    worst = int(np.argmax(dist - allowed))
    assert np.all(dist <= allowed), (
        f"code mismatch away from a rounding tie at row {r[worst]}, column {c[worst]}: oracle value "
        f"{yr[worst]!r} is {dist[worst]:.3e} from the boundary {b_r[worst]!r}, allowed {allowed[worst]:.3e}")
    return frac, float((dist / np.maximum(allowed, 1e-300)).max())
