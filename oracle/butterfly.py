"""Float64 oracle of the learnable orthogonal butterfly transform.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

The method (ButterflyQuant abstract, arXiv 2509.09679; explainer article,
section "butterfly") replaces a fixed Hadamard rotation by a butterfly of
Givens rotations whose angles are continuous parameters, so that Q is
orthogonal by construction, costs O(n log n) to apply and carries n*log2(n)/2
angles.  Rotating activations and weights with the same Q leaves a linear
layer unchanged: y = W x = (W Q^T)(Q x)  (abstract, computational invariance).

Notation and the readings this module takes where the pages are silent:

* width m = 2**L, L stages s = 0 .. L-1;
* stage s rotates every index pair (i, j = i + 2**s) with bit s of i clear,
  using the pair number p = ((i >> (s+1)) << s) | (i & (2**s - 1)) and the
  angle theta[s, p]  (angle array shape (L, m/2); flat index s*(m/2) + p);
* one rotation is  y_i = c*x_i - s*x_j,  y_j = s*x_i + c*x_j  with
  c = cos(theta), s = sin(theta);
* stage order (not fixed by the pages): Q = B_{L-1} ... B_1 B_0, i.e. stage 0
  (stride 1) acts first;
* Kronecker composite for n = m*r (explainer article, section "butterfly":
  non-power-of-two widths such as 5120 use a Kronecker-product composite):
  Q = B_m (x) O_r with the textbook definition
  (A (x) B)[i1*r + i2, j1*r + j2] = A[i1, j1] * B[i2, j2], so B_m acts on the
  stride-r index i1 and the dense orthogonal O_r on contiguous groups of r;
* backward: the loss is taken linear in Y with upstream gradient dY, so
  dX = Q^T dY per token and, for each stage with output v and output-gradient
  g, d theta[s, p] = sum over tokens of (g_j v_i - g_i v_j)  (chain rule of the
  rotation above; stage inputs are recovered as B_s^T v, nothing is stored).

Angles are given as float32 arrays (the shared input); cos and sin are taken
in float64 of those float32 values.
"""

from __future__ import annotations

import numpy as np


def num_stages(m: int) -> int:
    """log2(m) for a power of two m >= 2 (the butterfly needs a power of two)."""
    if m < 2 or (m & (m - 1)) != 0:
        raise ValueError(f"butterfly width must be a power of two >= 2, got {m}")
    return m.bit_length() - 1


def num_angles(m: int) -> int:
    """Learnable parameter count n*log2(n)/2 (abstract: half of n log n angles are learned)."""
    return m * num_stages(m) // 2


def pair_indices(m: int, s: int):
    """Index pairs of stage s: arrays (i, j, p) with j = i + 2**s and bit s of i clear.

    p is the pair number used to look up theta[s, p]; pairs are listed in
    increasing i, which is also increasing p.
    """
    half = 1 << s
    i = np.array([k for k in range(m) if not (k >> s) & 1], dtype=np.int64)
    j = i + half
    p = ((i >> (s + 1)) << s) | (i & (half - 1))
    return i, j, p


def _cos_sin(theta_row):
    t = np.asarray(theta_row, dtype=np.float32).astype(np.float64)
    return np.cos(t), np.sin(t)


def _check_theta(theta, m):
    theta = np.asarray(theta)
    L = num_stages(m)
    if theta.shape != (L, m // 2):
        raise ValueError(f"theta must have shape {(L, m // 2)}, got {theta.shape}")
    return theta


def apply_stage(theta, x, s, transpose=False):
    """Apply B_s (or B_s^T) to every row of x (float64, shape (rows, m)); returns a new array."""
    m = x.shape[-1]
    i, j, p = pair_indices(m, s)
    c, sn = _cos_sin(theta[s][p])
    if transpose:
        sn = -sn
    xi = x[..., i]
    xj = x[..., j]
    y = np.empty_like(x)
    y[..., i] = c * xi - sn * xj
    y[..., j] = sn * xi + c * xj
    return y


def forward(theta, x):
    """y = Q x for every row of x: stages 0, 1, ..., L-1 in that order (float64)."""
    x = np.asarray(x, dtype=np.float64)
    m = x.shape[-1]
    theta = _check_theta(theta, m)
    for s in range(num_stages(m)):
        x = apply_stage(theta, x, s)
    return x


def hadamard_preset_forward(quadrant, x):
    """y = Q x for the Hadamard preset: rotation (s, p) at the angle pi/4 + k pi/2,
    k = quadrant[s][p] & 3 (quadrant None: k = 0 everywhere), with its cos and sin
    taken as exactly +-1/sqrt(2).  H_n is the butterfly at particular angles
    (explainer article, section "butterfly"); every entry of the result is
    +-1/sqrt(n)."""
    x = np.asarray(x, dtype=np.float64)
    m = x.shape[-1]
    r = 1.0 / np.sqrt(2.0)
    for s in range(num_stages(m)):
        i, j, p = pair_indices(m, s)
        k = np.zeros(len(p), dtype=np.int64) if quadrant is None else (np.asarray(quadrant)[s][p].astype(np.int64) & 3)
        c = np.where((k == 0) | (k == 3), r, -r)
        sn = np.where(k <= 1, r, -r)
        xi = x[..., i]
        xj = x[..., j]
        y = np.empty_like(x)
        y[..., i] = c * xi - sn * xj
        y[..., j] = sn * xi + c * xj
        x = y
    return x


def inverse(theta, y):
    """x = Q^T y: stages L-1, ..., 0 with every angle negated (Q is orthogonal)."""
    y = np.asarray(y, dtype=np.float64)
    m = y.shape[-1]
    theta = _check_theta(theta, m)
    for s in reversed(range(num_stages(m))):
        y = apply_stage(theta, y, s, transpose=True)
    return y


def stage_matrix(theta, m: int, s: int):
    """Dense m x m matrix of stage s, built entry by entry (independent of apply_stage)."""
    theta = _check_theta(theta, m)
    B = np.zeros((m, m), dtype=np.float64)
    half = 1 << s
    for i in range(m):
        if (i >> s) & 1:
            continue
        j = i + half
        p = ((i >> (s + 1)) << s) | (i & (half - 1))
        t = float(np.float32(theta[s][p]))
        c, sn = np.cos(t), np.sin(t)
        B[i, i] = c
        B[i, j] = -sn
        B[j, i] = sn
        B[j, j] = c
    return B


def dense_q(theta, m: int):
    """Q = B_{L-1} ... B_1 B_0 as a dense matrix (product of explicit stage matrices)."""
    Q = np.eye(m)
    for s in range(num_stages(m)):
        Q = stage_matrix(theta, m, s) @ Q
    return Q


# ----------------------------------------------------------------------------
# Kronecker composite  Q = B_m (x) O_r  (n = m * r)
# ----------------------------------------------------------------------------

def _split(x, m, r):
    x = np.asarray(x, dtype=np.float64)
    if x.shape[-1] != m * r:
        raise ValueError(f"row width {x.shape[-1]} != m*r = {m * r}")
    return x.reshape(x.shape[:-1] + (m, r))


def kron_forward(theta, O, x, m: int):
    """y = (B_m (x) O_r) x per row.

    x[..., i1*r + i2] is viewed as a (m, r) array; O_r acts on the contiguous
    axis i2 and the butterfly on the strided axis i1.  The two factors commute.
    """
    O = np.asarray(O, dtype=np.float64)
    r = O.shape[0]
    v = _split(x, m, r)
    v = v @ O.T                              # O on each contiguous group of r
    v = np.swapaxes(v, -1, -2)               # (..., r, m): one length-m sub-row per i2
    v = forward(theta, v)
    v = np.swapaxes(v, -1, -2)
    return v.reshape(v.shape[:-2] + (m * r,))


def kron_inverse(theta, O, y, m: int):
    """x = (B_m (x) O_r)^T y = (B_m^T (x) O_r^T) y per row."""
    O = np.asarray(O, dtype=np.float64)
    r = O.shape[0]
    v = _split(y, m, r)
    v = np.swapaxes(v, -1, -2)
    v = inverse(theta, v)
    v = np.swapaxes(v, -1, -2)
    v = v @ O                                # O^T applied to each group
    return v.reshape(v.shape[:-2] + (m * r,))


def dense_kron_q(theta, O, m: int):
    """Dense (m*r) x (m*r) composite matrix via numpy.kron (for small tests)."""
    return np.kron(dense_q(theta, m), np.asarray(O, dtype=np.float64))


# ----------------------------------------------------------------------------
# Backward (calibration): dX = Q^T dY and dtheta summed over tokens
# ----------------------------------------------------------------------------

def backward(theta, x, dy):
    """Return (y, dx, dtheta) for y = Q x with the loss linear in y.

    dtheta has the angle layout (L, m/2) and is the sum over all rows.  The
    reverse sweep walks from v = y, g = dy through stages L-1 .. 0:
        dtheta[s, p] += g_j * v_i - g_i * v_j
        g <- B_s^T g ;  v <- B_s^T v
    and ends with dx = g.
    """
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    m = x.shape[-1]
    theta = _check_theta(theta, m)
    L = num_stages(m)
    y = forward(theta, x)
    v = y.reshape(-1, m)
    g = dy.reshape(-1, m)
    dtheta = np.zeros((L, m // 2), dtype=np.float64)
    for s in reversed(range(L)):
        i, j, p = pair_indices(m, s)
        contrib = g[:, j] * v[:, i] - g[:, i] * v[:, j]
        dtheta[s, p] += contrib.sum(axis=0)
        g = apply_stage(theta, g, s, transpose=True)
        v = apply_stage(theta, v, s, transpose=True)
    return y, g.reshape(dy.shape), dtheta


def backward_abs_scale(theta, x, dy):
    """A[s, p] = sum over rows of |g_j v_i| + |g_i v_j| (the size of the terms summed into dtheta).

    Used to scale the dtheta tolerance: floating-point error of a sum is
    bounded relative to the sum of the absolute values of its terms.
    """
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    m = x.shape[-1]
    theta = _check_theta(theta, m)
    L = num_stages(m)
    v = forward(theta, x).reshape(-1, m)
    g = dy.reshape(-1, m)
    A = np.zeros((L, m // 2), dtype=np.float64)
    for s in reversed(range(L)):
        i, j, p = pair_indices(m, s)
        A[s, p] += (np.abs(g[:, j] * v[:, i]) + np.abs(g[:, i] * v[:, j])).sum(axis=0)
        g = apply_stage(theta, g, s, transpose=True)
        v = apply_stage(theta, v, s, transpose=True)
    return A


def kron_backward(theta, O, x, dy, m: int):
    """(y, dx, dtheta) for the composite y = (B_m (x) O_r) x with fixed O_r.

    O_r is an input (not learned); dtheta collects the butterfly angles over
    every token and every one of the r interleaved sub-rows.
    """
    O = np.asarray(O, dtype=np.float64)
    r = O.shape[0]
    xo = _split(x, m, r) @ O.T                                   # (I (x) O) x
    sub = np.swapaxes(xo, -1, -2).reshape(-1, m)                  # sub-rows along i1
    dsub = np.swapaxes(_split(dy, m, r), -1, -2).reshape(-1, m)
    ysub, gsub, dtheta = backward(theta, sub, dsub)
    lead = np.asarray(x).shape[:-1]
    y = np.swapaxes(ysub.reshape(lead + (r, m)), -1, -2).reshape(lead + (m * r,))
    g = np.swapaxes(gsub.reshape(lead + (r, m)), -1, -2)          # (..., m, r)
    dx = (g @ O).reshape(lead + (m * r,))                          # (I (x) O^T) g
    return y, dx, dtheta
