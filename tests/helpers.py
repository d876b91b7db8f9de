"""Shared helpers of the GPU parity tests: device transfers and the comparison rules.

Comparison rules (per the accuracy bounds of the transform path):
* float32 outputs: per row, max |y_gpu - y_oracle| <= 2e-5 * ||x||_2;
* bfloat16 outputs: bitwise the round-to-nearest-even of the GPU's own float32
  output, and within one bf16 ulp of the oracle plus the float32 bound (a
  literal one-ulp bound is unreachable for elements much smaller than 2e-5 ||x||);
* quantized codes, scales and zero points computed from identical float32
  inputs are bit-exact; end to end, codes may differ by one level in at most
  1e-4 of the entries;
* dtheta: |gpu - oracle| <= 2e-4 * A + 1e-6 * max(A), A = sum of |terms|.
"""

from __future__ import annotations

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
