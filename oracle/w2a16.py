"""Float64 oracle of the W2A16 consumer GEMM: the rotated activations times the
dequantized rotated weights.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages deploy the transform with 2-bit weights and 16-bit activations
(explainer article, section "training & results": W2A16), and the layer's output
is unchanged by the rotation because y = W x = (W Q^T)(Q x) (ButterflyQuant
abstract).  The quantized layer therefore multiplies the 16-bit activations
x~ = Q x by the dequantized codes of W Q^T.  The pages print no kernel; the
readings taken here:

1. the weights arrive as ``quant``'s packed codes with fp16 scale and zero
   point per group (what bq_weight_rotate_pack writes); 4-bit codes use the same
   rules (W4A16);
2. a weight is dequantized as w_hat = (q - z) * s in float32, which is exact
   (an integer of at most 5 bits times an fp16 value), and enters the 16-bit
   product in the activations' type, bfloat16, rounded to nearest even;
3. the activations are bfloat16 values (Q x rounded to bfloat16);
4. out[t][o] = sum_k x~[t][k] * bf16(w_hat[o][k]).  Each product of two
   bfloat16 values is exact in float64 and the sum of K of them carries a
   relative error of at most K * 2^-53, so this is the exact result for every
   tolerance the float32 GPU accumulation needs.
"""

from __future__ import annotations

import numpy as np

from . import quant as oq


def bf16_round(x) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); the result is
    returned as float32 values that are exactly representable in bfloat16.
    NaN stays NaN; values beyond the largest bfloat16 round to infinity."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    out = rounded.view(np.float32).copy()
    nan = np.isnan(x)
    out[nan] = np.float32("nan")
    return out


def dequantize_bf16(codes_packed, scale16, zero16, bits: int, group: int, n: int) -> np.ndarray:
    """bf16(w_hat) as float32 values, (rows, n), from packed codes and fp16 bit patterns."""
    q = oq.unpack(np.asarray(codes_packed, dtype=np.uint8), bits, n)
    return bf16_round(oq.dequantize(q, scale16, zero16, group))


def w2a16_gemm(x_bf16, codes_packed, scale16, zero16, bits: int, group: int):
    """(out, sum_abs) in float64, both (tokens, out_features).

    x_bf16: (tokens, n) bfloat16 values held as float32 (or float64) numbers.
    sum_abs[t][o] = sum_k |x~[t][k] * w[o][k]|, the scale of the rounding error of
    any order of summation (used for tolerances)."""
    x = np.asarray(x_bf16, dtype=np.float64)
    n = x.shape[1]
    w = dequantize_bf16(codes_packed, scale16, zero16, bits, group, n).astype(np.float64)
    return x @ w.T, np.abs(x) @ np.abs(w).T
