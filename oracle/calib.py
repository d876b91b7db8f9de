"""Float64 oracle of the calibration losses: the uniformity regulariser and the
reconstruction loss with a straight-through estimator.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The angles are learned with a loss that includes a uniformity regularisation of
the post-transformation activations (ButterflyQuant abstract): the KL divergence
between the distribution of the rotated activations and the uniform
distribution over the quantization intervals, which pushes the transform to
spread activations evenly over the levels of the quantizer (explainer article,
section "training & results").  The pages give no estimator, smoothing or
weighting.  The readings taken here:

1. the bins of a group are the qmax + 1 levels of the group's own RTN grid: the
   scale s and zero point z come from the quantizer (``quant.group_params``,
   float32 steps on the float32 activations), and u = y / s + z is the real-valued
   position of y on that grid;
2. u is clamped to [0, qmax] and spread over the two nearest levels with a
   triangular kernel, w_c = max(0, 1 - |u - c|): the soft histogram of a group
   is p_c = (1/g) sum_i w_c(u_i), which sums to one;
3. p is smoothed, p~_c = (p_c + eps) / (1 + B eps) with B = qmax + 1, so that
   empty levels have a finite logarithm;
4. the loss is the mean over all groups of all rows of KL(p~ || uniform) =
   sum_c p~_c log(B p~_c);
5. the gradient treats s and z as constants (they come from the group's min
   and max), and a value with u outside (0, qmax) has zero gradient.  For u in
   (k, k+1) only w_k and w_{k+1} move, so
       dL/dy = (log p~_{k+1} - log p~_k) / (s g G (1 + B eps))
   with G the number of groups (the +1 of d(p log p) cancels).
"""

from __future__ import annotations

import numpy as np

from . import quant as oq


def soft_histogram(y32, bits: int, group: int):
    """(p, u, s) per group: p (rows, G, B) soft histogram, u (rows, G, g) the clamped
    grid positions in float64, s (rows, G) float32 scales."""
    y32 = np.asarray(y32, dtype=np.float32)
    rows, n = y32.shape
    _, _, s, z = oq.group_params(y32, bits, group)
    qmax = 2 ** bits - 1
    B = qmax + 1
    v = y32.reshape(rows, n // group, group).astype(np.float64)
    u = v / s.astype(np.float64)[..., None] + z.astype(np.float64)[..., None]
    uc = np.clip(u, 0.0, float(qmax))
    p = np.zeros((rows, n // group, B))
    for c in range(B):
        p[..., c] = np.maximum(0.0, 1.0 - np.abs(uc - c)).sum(axis=-1) / group
    return p, u, s


def uniformity_loss(y32, bits: int, group: int, eps: float):
    """(loss, kl per group (rows, G), dloss/dy (rows, n)) in float64."""
    y32 = np.asarray(y32, dtype=np.float32)
    rows, n = y32.shape
    qmax = 2 ** bits - 1
    B = qmax + 1
    G = rows * (n // group)
    p, u, s = soft_histogram(y32, bits, group)
    pt = (p + eps) / (1.0 + B * eps)
    logs = np.log(B * pt)
    kl = (pt * logs).sum(axis=-1)
    loss = kl.mean()
    # gradient: only the two levels around u move, with slopes -1 and +1
    inside = (u > 0.0) & (u < qmax)
    k = np.clip(np.floor(u), 0, qmax - 1).astype(np.int64)
    lk = np.take_along_axis(logs, k, axis=-1)
    lk1 = np.take_along_axis(logs, k + 1, axis=-1)
    d = (lk1 - lk) / (s.astype(np.float64)[..., None] * group * G * (1.0 + B * eps))
    dy = np.where(inside, d, 0.0).reshape(rows, n)
    return loss, kl, dy


def reconstruction_loss(theta, w, x, bits: int, group: int, abs_scale: bool = False):
    """Reconstruction loss of one linear layer under weight quantization, and its
    gradient with a straight-through estimator (readings of the explainer article,
    section "training & results": the quantized layer's output should match the
    original one; the abstract's invariance y = W x = (W Q^T)(Q x)).

    V = W Q^T (row o of V is Q w_o), W_hat = dequantize(RTN(V)) with the quantizer
    of ``quant`` applied to V rounded to float32, x~ = Q x per token, and
        r[t, o] = (W_hat x~_t)_o - (W x_t)_o,   loss = (1/T) sum_t ||r_t||^2.
    The straight-through estimator takes dW_hat / dV as the identity, so
        G_x = dloss/dx~ = (2/T) r W_hat,   G_v = dloss/dV = (2/T) r^T x~,
    and dtheta adds the backward of the activation side (rows x, gradient G_x)
    and of the weight side (rows w, gradient G_v).  Returns (loss, dtheta), or with
    abs_scale=True (loss, dtheta, A) where A = the sizes of the terms summed into
    dtheta, both sides (``butterfly.backward_abs_scale``), which scales the tolerance
    of a float32 dtheta per angle."""
    from . import butterfly as ob
    w = np.asarray(w, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    v = ob.forward(theta, w)
    codes, scale16, zero16 = oq.quantize_codes(v.astype(np.float32), bits, group)
    w_hat = oq.dequantize(codes, scale16, zero16, group).astype(np.float64)
    xt = ob.forward(theta, x)
    r = xt @ w_hat.T - x @ w.T
    loss = float((r * r).sum() / T)
    g_x = (2.0 / T) * (r @ w_hat)
    g_v = (2.0 / T) * (r.T @ xt)
    _, _, dth_x = ob.backward(theta, x, g_x)
    _, _, dth_v = ob.backward(theta, w, g_v)
    if abs_scale:
        A = ob.backward_abs_scale(theta, x, g_x) + ob.backward_abs_scale(theta, w, g_v)
        return loss, dth_x + dth_v, A
    return loss, dth_x + dth_v
