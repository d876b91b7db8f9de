"""Parity of the uniformity regulariser (bq_uniformity_loss) with the float64 oracle,
and a short calibration loop (forward, regulariser gradient, backward, angle step)
that lowers the regulariser on synthetic activations with outlier channels."""

import numpy as np
import pytest

from oracle import calib as oc
from rotation_bit_quantization_b200 import workloads as wl
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bq():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import rotation_bit_quantization_b200 as bq_mod
    from rotation_bit_quantization_b200 import build
    build.build()
    bq_mod.load()
    return bq_mod


def _acts(seed, rows, n):
    rng = np.random.default_rng(seed)
    y = (rng.standard_t(3.0, (rows, n)) * 0.5).astype(np.float32)
    y[:, rng.choice(n, 6, replace=False)] *= 40.0          # outlier channels
    return y


def _run(bq, y, bits, group, eps):
    torch = H.torch()
    rows, n = y.shape
    yd = H.dev_f32(y)
    kl = torch.empty((rows, n // group), dtype=torch.float32, device="cuda")
    dy = torch.empty_like(yd)
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    bq.bq_uniformity_loss(yd, bits, group, eps, kl, dy, loss)
    torch.cuda.synchronize()
    return H.host(kl), H.host(dy), float(H.host(loss)[0])


@pytest.mark.parametrize("bits,group", [(2, 64), (2, 128), (4, 128), (4, 256), (4, 64), (2, 256)])
def test_uniformity_matches_oracle(bq, bits, group):
    eps = 1e-4
    y = _acts(bits * 100 + group, 37, 4096)
    kl, dy, loss = _run(bq, y, bits, group, eps)
    ref_loss, ref_kl, ref_dy = oc.uniformity_loss(y, bits, group, eps)
    assert np.abs(kl - ref_kl).max() <= 2e-5 * (1 + np.abs(ref_kl).max())
    assert abs(loss - ref_loss) <= 2e-5 * abs(ref_loss) + 1e-7
    # the gradient jumps where u crosses a level: compare where u is clearly between
    # two levels or clearly outside [0, qmax]
    _, u, _ = oc.soft_histogram(y, bits, group)
    u = u.reshape(y.shape)
    qmax = 2 ** bits - 1
    frac = u - np.floor(u)
    clear = ((frac > 1e-3) & (frac < 1 - 1e-3) & (u > 1e-3) & (u < qmax - 1e-3)) | (u < -1e-3) | (u > qmax + 1e-3)
    assert clear.mean() > 0.99
    scale = np.abs(ref_dy).max()
    err = np.abs(dy - ref_dy)[clear]
    assert np.all(err <= 1e-4 * scale + 1e-4 * np.abs(ref_dy)[clear]), err.max() / scale
    assert np.all(dy[(u < -1e-3) | (u > qmax + 1e-3)] == 0.0)
    kl2, dy2, loss2 = _run(bq, y, bits, group, eps)
    assert np.array_equal(kl, kl2) and np.array_equal(dy, dy2) and loss == loss2


def test_uniformity_small_rows_and_degenerate_groups(bq):
    y = _acts(7, 3, 1024)
    y[1, :128] = 2.5                      # a constant group: hi == lo
    y[2, 128:256] = 0.0
    kl, dy, loss = _run(bq, y, 4, 128, 1e-3)
    ref_loss, ref_kl, ref_dy = oc.uniformity_loss(y, 4, 128, 1e-3)
    assert np.abs(kl - ref_kl).max() <= 2e-5 * (1 + np.abs(ref_kl).max())
    assert abs(loss - ref_loss) <= 2e-5 * abs(ref_loss)


def test_uniformity_loss_mean_of_a_large_batch(bq):
    """4097 rows x 4096 at INT4 g128 (131 104 groups, eight slices with ragged
    tails): the loss is the mean of the returned per-group values (float64 sums
    on both sides, so within one float32 step), repeats bitwise, and sampled rows'
    per-group values match the oracle."""
    rows, n, bits, group, eps = 4097, 4096, 4, 128, 1e-4
    y = _acts(11, rows, n)
    kl, _, loss = _run(bq, y, bits, group, eps)
    mean = float(np.float32(kl.astype(np.float64).mean()))
    assert abs(loss - mean) <= np.spacing(np.float32(abs(mean)))
    kl2, _, loss2 = _run(bq, y, bits, group, eps)
    assert loss2 == loss and np.array_equal(kl, kl2)
    sample = np.array([0, 1, 2048, 4095, 4096])
    _, ref_kl, _ = oc.uniformity_loss(y[sample], bits, group, eps)
    assert np.abs(kl[sample] - ref_kl).max() <= 2e-5 * (1 + np.abs(ref_kl).max())


def test_calibration_steps_lower_the_regulariser(bq):
    """Forward -> regulariser gradient -> backward (dtheta) -> angle step, repeated:
    the butterfly learns a rotation that spreads the outlier channels over the
    quantizer's levels, so the regulariser must fall."""
    torch = H.torch()
    m, rows, bits, group, eps = 1024, 64, 4, 128, 1e-4
    rng = np.random.default_rng(3)
    theta = torch.from_numpy(wl.uniform_angles(rng, m)).cuda()
    x = _acts(4, rows, m)
    xd = H.dev_f32(x)[None]
    y = torch.empty((rows, m), dtype=torch.float32, device="cuda")
    kl = torch.empty((rows, m // group), dtype=torch.float32, device="cuda")
    dy = torch.empty_like(y)
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    ybwd = torch.empty((1, rows, m), dtype=torch.float32, device="cuda")
    dx = torch.empty((1, rows, m), dtype=torch.float32, device="cuda")
    dth = torch.empty((1, theta.numel()), dtype=torch.float32, device="cuda")
    ws = torch.empty(bq.bq_butterfly_bwd_workspace_size(m, 1, rows), dtype=torch.uint8, device="cuda")
    losses = []
    for step in range(12):
        layer = bq.Layer(theta)
        bq.bq_butterfly_fwd(layer, xd[0], y)
        bq.bq_uniformity_loss(y, bits, group, eps, kl, dy, loss)
        bq.bq_butterfly_bwd([layer], xd, ybwd, dy[None], dx, dth, ws)
        torch.cuda.synchronize()
        losses.append(float(loss.item()))
        lr = 0.02 / float(dth.abs().max().item())      # at most 0.02 rad per angle and step
        bq.bq_angle_sgd(theta, dth.view(theta.shape), lr)
    assert losses[-1] < 0.9 * losses[0], losses
    assert all(np.isfinite(losses))


# --------------------------------------------------------------------------- reconstruction loss

def _recon_gpu(bq, theta, w, x, bits, group):
    torch = H.torch()
    n = w.shape[1]
    layer = bq.Layer(H.dev_f32(theta))
    ws = torch.empty(bq.bq_reconstruction_workspace_size(n, w.shape[0], x.shape[0], bits, group),
                     dtype=torch.uint8, device="cuda")
    dth = torch.empty(theta.size, dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    bq.bq_reconstruction_loss(layer, H.dev_f32(w), H.dev_f32(x), bits, group, dth, loss, ws)
    torch.cuda.synchronize()
    return float(H.host(loss)[0]), H.host(dth).reshape(theta.shape), layer


@pytest.mark.parametrize("m,out,T,bits,group", [(256, 48, 40, 2, 64), (1024, 40, 33, 4, 128), (4096, 96, 64, 2, 128)])
def test_reconstruction_matches_oracle(bq, m, out, T, bits, group):
    torch = H.torch()
    rng = np.random.default_rng(m + out + T)
    theta = wl.uniform_angles(rng, m)
    w = (rng.standard_normal((out, m)) * 0.02).astype(np.float32)
    w[:, rng.choice(m, max(1, m // 100), replace=False)] *= 10.0
    x = _acts(m + 1, T, m)
    loss, dth, layer = _recon_gpu(bq, theta, w, x, bits, group)
    # the codes the GPU quantized (bitwise the quantizer on its float32 forward) equal the
    # oracle's own codes here, so the two losses see the same W_hat
    from oracle import butterfly as ob
    from oracle import quant as oq
    codes, _, _ = bq.quant_outputs(out, m, bits, group, "cuda")
    c_gpu = torch.empty_like(codes); sc = torch.empty((out, m // group), dtype=torch.int16, device="cuda")
    zc = torch.empty_like(sc)
    bq.bq_weight_rotate_pack(layer, H.dev_f32(w), bits, group, c_gpu, sc, zc)
    torch.cuda.synchronize()
    c_ref, _, _ = oq.quantize_pack(ob.forward(theta, w.astype(np.float64)).astype(np.float32), bits, group)
    assert np.array_equal(H.host(c_gpu), c_ref)
    ref_loss, ref_dth, A = oc.reconstruction_loss(theta, w, x, bits, group, abs_scale=True)
    assert abs(loss - ref_loss) <= 2e-4 * ref_loss
    # per angle, scaled by the size of the terms summed into it (as for the plain backward)
    err = np.abs(dth - ref_dth)
    bound = 2e-4 * A + 1e-6 * A.max()
    assert np.all(err <= bound), f"dtheta error {np.max(err / bound):.2f} x the per-angle bound"
    loss2, dth2, _ = _recon_gpu(bq, theta, w, x, bits, group)
    assert loss2 == loss and np.array_equal(dth2, dth)


def test_calibration_steps_lower_the_reconstruction_loss(bq):
    """Angle steps on the straight-through gradient lower the W2A16 reconstruction
    loss of a layer whose activations carry outlier channels."""
    torch = H.torch()
    m, out, T, bits, group = 256, 64, 96, 2, 64
    rng = np.random.default_rng(8)
    theta = torch.from_numpy(wl.uniform_angles(rng, m)).cuda()
    w = H.dev_f32((rng.standard_normal((out, m)) * 0.02).astype(np.float32))
    x = H.dev_f32(_acts(9, T, m))
    ws = torch.empty(bq.bq_reconstruction_workspace_size(m, out, T, bits, group), dtype=torch.uint8, device="cuda")
    dth = torch.empty(theta.numel(), dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    losses = []
    for step in range(15):
        layer = bq.Layer(theta)
        bq.bq_reconstruction_loss(layer, w, x, bits, group, dth, loss, ws)
        torch.cuda.synchronize()
        losses.append(float(loss.item()))
        lr = 0.02 / float(dth.abs().max().item())
        bq.bq_angle_sgd(theta, dth.view(theta.shape), lr)
    assert min(losses[-3:]) < 0.9 * losses[0], losses


def test_calibration_from_the_hadamard_preset_beats_it(bq):
    """The method's claim on a synthetic layer: starting from the fixed Hadamard
    rotation (QuaRot's transform, the butterfly at pi/4), gradient steps on the W2A16
    reconstruction loss find angles with a lower loss than the Hadamard's own.  The
    layer's weights carry a few outlier input channels that the fixed rotation spreads
    but cannot adapt to."""
    torch = H.torch()
    m, out, T, bits, group = 256, 64, 128, 2, 64
    rng = np.random.default_rng(17)
    w = (rng.standard_normal((out, m)) * 0.02).astype(np.float32)
    w[:, rng.choice(m, 4, replace=False)] *= 12.0
    x = _acts(18, T, m)
    had = bq.Layer.hadamard(m)
    theta = had.theta.clone()
    wd, xd = H.dev_f32(w), H.dev_f32(x)
    ws = torch.empty(bq.bq_reconstruction_workspace_size(m, out, T, bits, group), dtype=torch.uint8, device="cuda")
    dth = torch.empty(theta.numel(), dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    losses = []
    for step in range(40):
        layer = bq.Layer(theta)
        bq.bq_reconstruction_loss(layer, wd, xd, bits, group, dth, loss, ws)
        torch.cuda.synchronize()
        losses.append(float(loss.item()))
        lr = 0.01 / float(dth.abs().max().item())
        bq.bq_angle_sgd(theta, dth.view(theta.shape), lr)
    # the first loss is the Hadamard preset's (its angles are pi/4 in float32)
    ref_loss, _ = oc.reconstruction_loss(np.full((8, m // 2), np.pi / 4, dtype=np.float32), w, x, bits, group)
    assert abs(losses[0] - ref_loss) <= 2e-4 * ref_loss
    assert min(losses[-5:]) < 0.9 * losses[0], losses
