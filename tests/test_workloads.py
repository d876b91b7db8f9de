"""The seeded input generators match the recipe stated for each workload: shapes,
dtypes, value ranges, the outlier channels and their sign, the bf16 conversion, and
determinism (the same call gives the same bytes).  Small row counts; no GPU."""

import numpy as np
import pytest

from rotation_bit_quantization_b200 import workloads as wl


def test_bf16_conversion_matches_the_library_and_widens_exactly():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    x = np.concatenate([
        (rng.standard_normal(20000) * 300.0).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),               # subnormals
        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8),   # exact ties to even
                  0.0, -0.0, np.inf, -np.inf, 3.3895314e38], dtype=np.float32),
    ]).astype(np.float32)
    bits = wl.bf16_bits_from_f32(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)
    widened = wl.f32_from_bf16_bits(bits)
    assert np.array_equal(widened, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())
    assert np.isnan(wl.f32_from_bf16_bits(wl.bf16_bits_from_f32(np.array([np.nan], np.float32))))[0]


@pytest.mark.parametrize("m", [2, 256, 1024, 4096])
def test_angles_shape_range_and_determinism(m):
    t = wl.uniform_angles(np.random.default_rng([2, 0]), m)
    assert t.dtype == np.float32 and t.shape == (m.bit_length() - 1, m // 2)
    assert np.all(t >= np.float32(-np.pi)) and np.all(t <= np.float32(np.pi))
    assert np.array_equal(t, wl.uniform_angles(np.random.default_rng([2, 0]), m))
    if t.size > 1000:
        assert abs(float(t.mean())) < 0.1 and t.min() < -3.0 and t.max() > 3.0


@pytest.mark.parametrize("r", [2, 3, 5, 8])
def test_random_orthogonal(r):
    O = wl.random_orthogonal(np.random.default_rng([4, 3]), r)
    assert O.dtype == np.float32 and O.shape == (r, r)
    eye = O.astype(np.float64) @ O.astype(np.float64).T
    assert np.abs(eye - np.eye(r)).max() < 1e-6
    # QR with diag(R) > 0 fixes the column signs: the same matrix from the same seed
    assert np.array_equal(O, wl.random_orthogonal(np.random.default_rng([4, 3]), r))


def _check_outliers(x_f32, ch, sign, factor_min):
    rest = np.delete(x_f32, ch, axis=1)
    big = np.abs(x_f32[:, ch])
    assert np.median(big) > factor_min * np.median(np.abs(rest))
    if sign > 0:
        assert np.all(x_f32[:, ch] >= 0)
    elif sign < 0:
        assert np.all(x_f32[:, ch] <= 0)


def test_act_4096():
    w = wl.act_4096(rows=64)
    assert (w.m, w.r, w.n, w.bits, w.group, w.x_dtype) == (4096, 1, 4096, 4, 128, "bf16")
    assert w.x.dtype == np.uint16 and w.x.shape == (64, 4096) and w.theta.shape == (12, 2048)
    ch = np.array(w.meta["outlier_channels"])
    assert len(ch) == 8 and np.all(np.diff(ch) > 0)
    _check_outliers(wl.f32_from_bf16_bits(w.x), ch, +1, 20.0)
    again = wl.act_4096(rows=64)
    assert np.array_equal(w.x, again.x) and np.array_equal(w.theta, again.theta)
    shifted = wl.act_4096(rows=64, seed_offset=1)           # another rank's batch: new X, same layer
    assert not np.array_equal(w.x, shifted.x) and np.array_equal(w.theta, shifted.theta)
    assert shifted.meta["outlier_channels"] == w.meta["outlier_channels"]


def test_weight_4096():
    w = wl.weight_4096(rows=64)
    assert (w.bits, w.group, w.w_dtype) == (2, 128, "bf16") and w.w.shape == (64, 4096)
    ch = np.array(w.meta["outlier_channels"])
    assert len(ch) == round(0.01 * 4096) == 41
    wf = wl.f32_from_bf16_bits(w.w)
    _check_outliers(wf, ch, 0, 5.0)
    assert 0.015 < np.std(np.delete(wf, ch, axis=1)) < 0.025   # N(0, 0.02) off the outlier columns


def test_act_5120():
    w = wl.act_5120(rows=16)
    assert (w.m, w.r, w.n) == (1024, 5, 5120) and w.O.shape == (5, 5) and w.theta.shape == (10, 512)
    ch = np.array(w.meta["outlier_channels"])
    assert len(ch) == 10
    _check_outliers(wl.f32_from_bf16_bits(w.x), ch, -1, 20.0)


def test_tiny():
    w = wl.tiny()
    assert w.x.shape == (64, 256) and w.w.shape == (128, 256) and (w.bits, w.group) == (2, 64)
    assert np.array_equal(w.theta, wl.uniform_angles(np.random.default_rng(0), 256))
    ch = np.array(w.meta["outlier_channels"])
    assert len(ch) == 3
    _check_outliers(w.x, ch, 0, 5.0)


def test_backward_layer_host():
    a = wl.backward_layer_host(3, 8)
    b = wl.backward_layer_host(3, 8)
    assert a.x.shape == (8, 4096) and a.dy.shape == (8, 4096) and a.dy.dtype == np.float32
    assert np.array_equal(a.x, b.x) and np.array_equal(a.dy, b.dy)
    assert np.array_equal(a.theta, wl.backward_angles(4, 4096)[3])
    assert not np.array_equal(a.theta, wl.backward_layer_host(4, 8).theta)


@pytest.mark.parametrize("bits,group", [(2, 64), (2, 128), (4, 128), (4, 256)])
def test_packed_weights_ranges(bits, group):
    codes, s16, z16 = wl.packed_weights(np.random.default_rng(1), 300, 1024, bits, group)
    assert codes.dtype == np.uint8 and codes.shape == (300, 1024 * bits // 8)
    assert codes.min() == 0 and codes.max() == 255                 # uniform code bytes
    s = s16.view(np.float16).astype(np.float64)
    z = z16.view(np.float16).astype(np.float64)
    assert s.shape == z.shape == (300, 1024 // group)
    assert s.min() >= 2.0 ** -9 * (1 - 2.0 ** -10) and s.max() <= 2.0 ** -5 * (1 + 2.0 ** -10)
    assert np.all(z == np.round(z)) and z.min() >= 0 and z.max() <= 2 ** bits - 1
    assert set(np.unique(z).astype(int)) == set(range(2 ** bits))


def test_w2a16_layer():
    x, codes, s16, z16, bits, group = wl.w2a16_4096(tokens=32, out_features=256)
    assert x.dtype == np.uint16 and x.shape == (32, 4096) and (bits, group) == (2, 128)
    assert codes.shape == (256, 1024) and s16.shape == z16.shape == (256, 32)
    again = wl.w2a16_4096(tokens=32, out_features=256)
    assert all(np.array_equal(u, v) for u, v in zip((x, codes, s16, z16), again[:4]))


def test_block_transforms_recipe():
    """Block transforms of the WUSH workload: (C/G, G, G) bf16 bits, I + 0.3 N(0,1)/sqrt(G) per
    block (diagonal near 1, off-diagonal spread 0.3/sqrt(G)), deterministic in the seed,
    different seeds and block sizes giving different matrices."""
    for C, G in ((4096, 32), (4096, 16), (320, 32)):
        Tb = wl.block_transforms(C, G, 7)
        assert Tb.shape == (C // G, G, G) and Tb.dtype == np.uint16
        T = wl.f32_from_bf16_bits(Tb).astype(np.float64)
        assert np.array_equal(wl.bf16_bits_from_f32(T.astype(np.float32)), Tb)   # bf16 values
        off = T - np.eye(G)[None]
        assert abs(off.std() - 0.3 / np.sqrt(G)) < 0.1 * 0.3 / np.sqrt(G)
        assert abs(np.diagonal(T, axis1=1, axis2=2).mean() - 1.0) < 0.02
        assert np.array_equal(wl.block_transforms(C, G, 7), Tb)
        assert not np.array_equal(wl.block_transforms(C, G, 8), Tb)
