"""Pins of the uniformity-regulariser oracle (oracle/calib.py) against what fixes it
independently of its own formulas: central finite differences of the loss, a
histogram that is uniform by construction (KL = 0), a two-level histogram with a
closed-form KL, the sign of the gradient, and a planted mistake."""

import numpy as np

from oracle import calib as oc
from oracle import quant as oq


def _fd_case(bits, group, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((2, 2 * group)) * 1.5).astype(np.float32)


def _fd_check(y, bits, group, eps, dy_fn):
    """Central differences on elements whose grid position is away from a level and
    that are not a group's min or max (s and z stay fixed)."""
    loss, _, dy = oc.uniformity_loss(y, bits, group, eps)
    _, u, s = oc.soft_histogram(y, bits, group)
    qmax = 2 ** bits - 1
    rows, n = y.shape
    uf = u.reshape(rows, n)
    g = y.reshape(rows, n // group, group)
    checked = 0
    for r in range(rows):
        for i in range(n):
            frac = uf[r, i] - np.floor(uf[r, i])
            grp = g[r, i // group]
            if not (0.1 < frac < 0.9) or not (0.5 < uf[r, i] < qmax - 0.5):
                continue
            if y[r, i] in (grp.min(), grp.max()):
                continue
            h = np.float32(0.01) * np.float32(s[r, i // group])
            yp, ym = y.copy(), y.copy()
            yp[r, i] = np.float32(y[r, i] + h)
            ym[r, i] = np.float32(y[r, i] - h)
            fd = (oc.uniformity_loss(yp, bits, group, eps)[0] - oc.uniformity_loss(ym, bits, group, eps)[0]) / (
                float(yp[r, i]) - float(ym[r, i]))
            assert abs(fd - dy_fn(dy)[r, i]) <= 1e-6 * max(1.0, abs(fd)) + 1e-3 * abs(fd), (r, i, fd, dy[r, i])
            checked += 1
    assert checked >= 10
    return loss


def test_gradient_matches_finite_differences():
    for bits, group in ((2, 32), (4, 64)):
        y = _fd_case(bits, group, bits + group)
        _fd_check(y, bits, group, 1e-4, lambda d: d)


def test_planted_dropped_scale_is_caught():
    bits, group = 2, 32
    y = _fd_case(bits, group, 5)
    _, _, s = oc.soft_histogram(y, bits, group)
    assert np.all(np.abs(s - 1) > 0.05)
    try:
        # the gradient without its 1/s factor
        _fd_check(y, bits, group, 1e-4, lambda d: d * np.repeat(s, group, axis=1))
    except AssertionError:
        return
    raise AssertionError("a gradient missing 1/s passed the finite-difference pin")


def test_uniform_histogram_has_zero_kl_and_gradient():
    # s = 0.5, z = 1 (both exact): 16 values on each of the 4 levels of an INT2 grid
    s, z = 0.5, 1
    levels = np.array([(c - z) * s for c in range(4)], np.float32)
    y = np.repeat(levels, 16)[None, :].astype(np.float32)
    np.random.default_rng(0).shuffle(y[0])
    scale16, zero16, s32, z32 = oq.group_params(y, 2, 64)
    assert s32[0, 0] == np.float32(s) and z32[0, 0] == np.float32(z)
    loss, kl, dy = oc.uniformity_loss(y, 2, 64, 1e-4)
    assert abs(loss) < 1e-15 and np.all(np.abs(dy) < 1e-15)


def test_two_level_histogram_closed_form():
    # half the group on the bottom level, half on the top: p = (1/2, 0, ..., 0, 1/2)
    for bits in (2, 4):
        qmax = 2 ** bits - 1
        B, eps = qmax + 1, 1e-3
        y = np.array([[0.0] * 32 + [float(qmax) * 0.25] * 32], np.float32)   # s = 0.25 exactly, z = 0
        loss, kl, dy = oc.uniformity_loss(y, bits, 64, eps)
        p = np.zeros(B); p[0] = p[-1] = 0.5
        pt = (p + eps) / (1 + B * eps)
        assert abs(loss - float((pt * np.log(B * pt)).sum())) < 1e-12
        assert np.all(dy == 0.0)          # every value sits at u = 0 or u = qmax


def test_gradient_points_toward_emptier_levels():
    # most of the group on level 0, one value between levels 0 and 1: raising it
    # moves mass to the emptier level 1, so the loss must fall (dL/dy < 0)
    y = np.array([[0.0] * 60 + [0.3, 3.0, 3.0, 3.0]], np.float32)            # s = 1, z = 0
    loss, kl, dy = oc.uniformity_loss(y, 2, 64, 1e-4)
    assert dy[0, 60] < 0


# --------------------------------------------------------------------------- reconstruction loss

from oracle import butterfly as ob                    # noqa: E402
from rotation_bit_quantization_b200 import workloads as wl  # noqa: E402


def _recon_case(seed, m=16, out=12, T=9):
    rng = np.random.default_rng(seed)
    theta = wl.uniform_angles(rng, m)
    w = rng.standard_normal((out, m)).astype(np.float32)
    x = rng.standard_normal((T, m)).astype(np.float32)
    return theta, w, x


def _q64(th64, m):
    """Dense Q from float64 angles (stage matrices), for finite differences in theta."""
    q = np.eye(m)
    for s in range(ob.num_stages(m)):
        B = np.zeros((m, m))
        half = 1 << s
        for i in range(m):
            if (i >> s) & 1:
                continue
            j = i + half
            p = ((i >> (s + 1)) << s) | (i & (half - 1))
            c, sn = np.cos(th64[s, p]), np.sin(th64[s, p])
            B[i, i], B[i, j], B[j, i], B[j, j] = c, -sn, sn, c
        q = B @ q
    return q


def _surrogate(th64, theta0, w, x, bits, group):
    """The straight-through surrogate around theta0: W_hat(theta) = RTN(V0) + V(theta) - V0."""
    m = w.shape[1]
    w64, x64 = w.astype(np.float64), x.astype(np.float64)
    v0 = ob.forward(theta0, w64)
    codes, s16, z16 = oq.quantize_codes(v0.astype(np.float32), bits, group)
    q = _q64(th64, m)
    w_hat = oq.dequantize(codes, s16, z16, group).astype(np.float64) + w64 @ q.T - v0
    r = (x64 @ q.T) @ w_hat.T - x64 @ w64.T
    return (r * r).sum() / x.shape[0]


def test_reconstruction_gradient_matches_surrogate_finite_differences():
    theta, w, x = _recon_case(1)
    loss, dth = oc.reconstruction_loss(theta, w, x, 2, 8)
    th0 = theta.astype(np.float64)
    assert abs(_surrogate(th0, theta, w, x, 2, 8) - loss) < 1e-10 * max(1.0, loss)
    h = 1e-6
    for s, p in ((0, 0), (1, 3), (2, 5), (3, 7)):
        tp, tm = th0.copy(), th0.copy()
        tp[s, p] += h
        tm[s, p] -= h
        fd = (_surrogate(tp, theta, w, x, 2, 8) - _surrogate(tm, theta, w, x, 2, 8)) / (2 * h)
        assert abs(fd - dth[s, p]) <= 1e-6 * max(1.0, abs(fd)), (s, p, fd, dth[s, p])


def test_reconstruction_planted_missing_weight_side_is_caught():
    theta, w, x = _recon_case(2)
    th0 = theta.astype(np.float64)
    v = ob.forward(theta, w.astype(np.float64))
    codes, s16, z16 = oq.quantize_codes(v.astype(np.float32), 2, 8)
    w_hat = oq.dequantize(codes, s16, z16, 8).astype(np.float64)
    xt = ob.forward(theta, x.astype(np.float64))
    r = xt @ w_hat.T - x.astype(np.float64) @ w.astype(np.float64).T
    _, _, wrong = ob.backward(theta, x, (2.0 / x.shape[0]) * (r @ w_hat))      # weight side dropped
    h = 1e-6
    tp, tm = th0.copy(), th0.copy()
    tp[1, 2] += h
    tm[1, 2] -= h
    fd = (_surrogate(tp, theta, w, x, 2, 8) - _surrogate(tm, theta, w, x, 2, 8)) / (2 * h)
    assert abs(fd - wrong[1, 2]) > 1e-4 * max(1.0, abs(fd))


def test_reconstruction_is_zero_for_an_exactly_quantizable_layer():
    # theta = 0 (Q = I) and weights on their groups' RTN grids: W_hat = W, r = 0
    m, out, group = 16, 6, 8
    rng = np.random.default_rng(4)
    q = rng.integers(0, 4, (out, m))
    q[:, ::group] = 0
    q[:, 1::group] = 3                                  # each group spans the full grid
    w = ((q - 1) * 0.25).astype(np.float32)            # s = 0.25, z = 1 exactly
    x = rng.standard_normal((5, m)).astype(np.float32)
    theta = np.zeros((4, m // 2), np.float32)
    loss, dth = oc.reconstruction_loss(theta, w, x, 2, group)
    assert loss == 0.0 and np.all(dth == 0.0)
