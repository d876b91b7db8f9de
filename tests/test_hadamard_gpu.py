"""Parity of the Hadamard presets (bq_precompute_hadamard) run through the transform
kernels with the float64 oracle preset, exactness of the fixed-point-free path (every
output of a unit input is exactly +-2^-6 at n = 4096), the angles the preset reports,
the inverse, and the fused quantizer."""

import numpy as np
import pytest

from oracle import butterfly as ob
from oracle import quant as oq
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


def _quadrant(rng, m):
    L = m.bit_length() - 1
    return rng.integers(0, 4, size=(L, m // 2)).astype(np.uint8)


def _layer(bq, m, k):
    torch = H.torch()
    return bq.Layer.hadamard(m, None if k is None else torch.from_numpy(k).cuda())


@pytest.mark.parametrize("m,random", [(4096, False), (4096, True), (1024, True), (256, False), (64, True)])
def test_preset_forward_matches_oracle(bq, m, random):
    torch = H.torch()
    rng = np.random.default_rng(m + random)
    k = _quadrant(rng, m) if random else None
    layer = _layer(bq, m, k)
    assert layer.fast_form
    x = (rng.standard_normal((37, m)) * 2.0).astype(np.float32)
    x[:, rng.choice(m, 3, replace=False)] *= 50.0
    y = torch.empty((37, m), dtype=torch.float32, device="cuda")
    bq.bq_butterfly_fwd(layer, H.dev_f32(x), y)
    torch.cuda.synchronize()
    ref = ob.hadamard_preset_forward(k, x.astype(np.float64))
    H.assert_f32_close(H.host(y), ref, x.astype(np.float64))


@pytest.mark.parametrize("random", [False, True])
def test_preset_is_exact_on_unit_inputs(bq, random):
    """Coefficients +-1 and an output scale of exactly 2^-6: every output of e_j is +-2^-6."""
    torch = H.torch()
    m = 4096
    rng = np.random.default_rng(3)
    k = _quadrant(rng, m) if random else None
    layer = _layer(bq, m, k)
    cols = rng.choice(m, 64, replace=False)
    x = np.zeros((64, m), dtype=np.float32)
    x[np.arange(64), cols] = 1.0
    y = torch.empty((64, m), dtype=torch.float32, device="cuda")
    bq.bq_butterfly_fwd(layer, H.dev_f32(x), y)
    torch.cuda.synchronize()
    got = H.host(y)
    assert np.all(np.abs(got) == 2.0 ** -6)
    assert np.array_equal(got, ob.hadamard_preset_forward(k, x.astype(np.float64)).astype(np.float32))


def test_preset_reports_its_angles(bq):
    m = 1024
    k = _quadrant(np.random.default_rng(5), m)
    layer = _layer(bq, m, k)
    want = (np.pi / 4 + np.where(k < 2, k, k.astype(np.int64) - 4) * (np.pi / 2)).astype(np.float32)
    assert np.array_equal(H.host(layer.theta), want)
    # the general path on those float32 angles is the same transform to float32 accuracy
    torch = H.torch()
    x = np.random.default_rng(6).standard_normal((8, m)).astype(np.float32)
    general = bq.Layer(layer.theta)
    y1 = torch.empty((8, m), dtype=torch.float32, device="cuda")
    y2 = torch.empty_like(y1)
    bq.bq_butterfly_fwd(layer, H.dev_f32(x), y1)
    bq.bq_butterfly_fwd(general, H.dev_f32(x), y2)
    torch.cuda.synchronize()
    H.assert_f32_close(H.host(y1), H.host(y2).astype(np.float64), x.astype(np.float64))


def test_preset_inverse_and_kronecker(bq):
    torch = H.torch()
    rng = np.random.default_rng(9)
    m = 4096
    k = _quadrant(rng, m)
    layer = _layer(bq, m, k)
    x = rng.standard_normal((16, m)).astype(np.float32)
    y = torch.empty((16, m), dtype=torch.float32, device="cuda")
    xb = torch.empty_like(y)
    bq.bq_butterfly_fwd(layer, H.dev_f32(x), y)
    bq.bq_butterfly_inv(layer, y, xb)
    torch.cuda.synchronize()
    H.assert_f32_close(H.host(xb), x.astype(np.float64), x.astype(np.float64))
    # B_1024 preset (x) O_5 through the n = 5120 kernel
    O = wl.random_orthogonal(rng, 5)
    kb = _quadrant(rng, 1024)
    kl = bq.Layer.hadamard(1024, torch.from_numpy(kb).cuda(), O=torch.from_numpy(O).cuda())
    x5 = rng.standard_normal((12, 5120)).astype(np.float32)
    y5 = torch.empty((12, 5120), dtype=torch.float32, device="cuda")
    bq.bq_butterfly_fwd(kl, H.dev_f32(x5), y5)
    torch.cuda.synchronize()
    theta_b = (np.pi / 4 + np.where(kb < 2, kb, kb.astype(np.int64) - 4) * (np.pi / 2)).astype(np.float32)
    ref = ob.kron_forward(theta_b, O, x5.astype(np.float64), 1024)
    H.assert_f32_close(H.host(y5), ref, x5.astype(np.float64))


def test_preset_quantize_is_the_quantizer_of_its_forward(bq):
    """Fused codes = the library's quantizer on the preset's own float32 output (GPU
    against GPU, through the exact identity layer), and within one level of the oracle's
    codes on at most 1e-4 of the entries end to end."""
    torch = H.torch()
    m, rows, bits, group = 4096, 40, 2, 128
    rng = np.random.default_rng(12)
    k = _quadrant(rng, m)
    layer = _layer(bq, m, k)
    x = (rng.standard_normal((rows, m)) * 0.5).astype(np.float32)
    xd = H.dev_f32(x)
    y = torch.empty((rows, m), dtype=torch.float32, device="cuda")
    bq.bq_butterfly_fwd(layer, xd, y)
    codes, scale, zero = bq.quant_outputs(rows, m, bits, group, "cuda")
    bq.bq_transform_quantize(layer, xd, bits, group, codes, scale, zero)
    ident = bq.Layer(torch.zeros((12, m // 2), dtype=torch.float32, device="cuda"))
    c2, s2, z2 = bq.quant_outputs(rows, m, bits, group, "cuda")
    bq.bq_transform_quantize(ident, y, bits, group, c2, s2, z2)
    torch.cuda.synchronize()
    assert torch.equal(codes, c2) and torch.equal(scale, s2) and torch.equal(zero, z2)
    ref = ob.hadamard_preset_forward(k, x.astype(np.float64))
    q_ref, _, _ = oq.quantize_codes(ref.astype(np.float32), bits, group)
    d = H.ordered_diff_codes(oq.unpack(H.host(codes), bits, m), q_ref)
    assert d.max() <= 1 and (d > 0).mean() <= 1e-4
