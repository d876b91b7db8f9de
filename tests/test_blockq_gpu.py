"""Parity of the block transform + block quantizer kernel (bq_block_transform_quantize,
tcgen05 on the tensor cores) with the oracle in oracle/blockq.py.

* The transform alone (format none): float32 output within the accumulation bound of
  bf16 x bf16 products summed in float32 (at most one rounding per 16 of K plus one,
  relative to sum |T x|); bfloat16 output bitwise the rounding of the float32 output.
* Codes and scales from the kernel's own float32 transform output: bit-exact against
  the oracle's quantizer (MXFP4, NVFP4, INT4).
* End to end against the float64 transform: every differing code one grid step from
  the oracle's, on a small fraction of the entries.
"""

import numpy as np
import pytest

from oracle import blockq as ob
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


def _case(seed, rows, C, G, scale=1.0):
    rng = np.random.default_rng(seed)
    Tb = wl.block_transforms(C, G, seed)
    x = (rng.standard_normal((rows, C)) * scale).astype(np.float32)
    x[:, rng.choice(C, max(1, C // 64), replace=False)] *= 30.0      # outlier channels
    xb = wl.bf16_bits_from_f32(x)
    return Tb, xb


def _dev_T(Tb):
    return H.dev_bf16_bits(Tb.reshape(-1, Tb.shape[-1])).view(Tb.shape)


def _run(bq, Tb, xb, fmt, gscale=1.0, y_dtype=None):
    torch = H.torch()
    bt = bq.BlockTransform(_dev_T(Tb))
    x = H.dev_bf16_bits(xb)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if fmt == "none":
        y = torch.empty(x.shape, dtype=y_dtype or torch.float32, device="cuda")
        bq.bq_block_transform_quantize(bt, x, "none", y=y, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        return H.host(y)
    codes, scales = bq.block_outputs(x.shape[0], x.shape[1], fmt, "cuda")
    bq.bq_block_transform_quantize(bt, x, fmt, codes, scales, gscale=gscale, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    sc = H.host(scales)
    return H.host(codes), (sc.view(np.uint16) if fmt == "int4" else sc)


def _ref(Tb, xb):
    T = wl.f32_from_bf16_bits(Tb).astype(np.float64)
    x = wl.f32_from_bf16_bits(xb).astype(np.float64)
    return ob.block_transform(T, x), T, x


def _assert_transform_close(y, ref, T, x, G):
    rows, C = x.shape
    absum = np.einsum("rbk,bok->rbo", np.abs(x).reshape(rows, C // G, G), np.abs(T)).reshape(rows, C)
    bound = (G / 16 + 1) * 2.0 ** -23 * absum + 1e-30
    err = np.abs(np.asarray(y, np.float64) - ref)
    assert np.all(err <= bound), f"max err / bound {np.max(err / bound):.2f}"


@pytest.mark.parametrize("G", [16, 32])
@pytest.mark.parametrize("rows,C", [(1, 64), (37, 256), (128, 128), (300, 4096)])
def test_transform_float32(bq, G, rows, C):
    Tb, xb = _case(rows + C + G, rows, C, G)
    y = _run(bq, Tb, xb, "none")
    ref, T, x = _ref(Tb, xb)
    _assert_transform_close(y, ref, T, x, G)


def test_transform_bfloat16_is_rounding_of_float32(bq):
    torch = H.torch()
    Tb, xb = _case(3, 257, 512, 32)
    y32 = _run(bq, Tb, xb, "none")
    y16 = _run(bq, Tb, xb, "none", y_dtype=torch.bfloat16)
    assert np.array_equal(y16, wl.bf16_bits_from_f32(y32))


def _assert_codes_close(q_gpu, q_ref, fmt, max_frac):
    """End to end: differing codes are one grid step apart, on at most max_frac of entries."""
    if fmt == "int4":
        a, b = ob.unpack4(q_gpu, signed=True).astype(int), ob.unpack4(q_ref, signed=True).astype(int)
        step = np.abs(a - b)
    else:
        ca, cb = ob.unpack4(q_gpu), ob.unpack4(q_ref)
        # E2M1 grid index with the sign: -7..7 (both zeros at 0)
        ia = np.where(ca & 8, -(ca & 7).astype(int), (ca & 7).astype(int))
        ib = np.where(cb & 8, -(cb & 7).astype(int), (cb & 7).astype(int))
        step = np.abs(ia - ib)
    assert step.max(initial=0) <= 1
    assert (step > 0).mean() <= max_frac, f"{(step > 0).mean():.2e}"


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "int4"])
@pytest.mark.parametrize("rows,C", [(1, 64), (131, 512), (2048, 4096)])
def test_quantizer_bitwise_and_end_to_end(bq, fmt, rows, C):
    G = ob.FORMATS[fmt]
    Tb, xb = _case(rows * 7 + C + G, rows, C, G)
    gscale = 0.75 if fmt == "nvfp4" else 1.0
    codes, scales = _run(bq, Tb, xb, fmt, gscale=gscale)
    y32 = _run(bq, Tb, xb, "none").astype(np.float32)
    # the fused codes are bitwise the oracle's quantizer applied to the kernel's own transform
    c_ref, s_ref = ob.quantize(y32, fmt, gscale)
    assert np.array_equal(scales, s_ref), f"{fmt} scales differ"
    assert np.array_equal(codes, c_ref), f"{fmt} codes differ on {(codes != c_ref).mean():.2e} of bytes"
    # end to end against the float64 transform
    ref, T, x = _ref(Tb, xb)
    _assert_transform_close(y32, ref, T, x, G)
    c_e2e, _ = ob.quantize(ref.astype(np.float32), fmt, gscale)
    _assert_codes_close(codes, c_e2e, fmt, 2e-3)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "int4"])
def test_quantizer_edge_groups(bq, fmt):
    """Identity transforms put chosen values straight into the quantizer: all-zero groups,
    huge and tiny magnitudes, exact rounding ties, values that round to -0."""
    G = ob.FORMATS[fmt]
    C = 256
    Tb = np.broadcast_to(wl.bf16_bits_from_f32(np.eye(G, dtype=np.float32)), (C // G, G, G)).copy()
    rng = np.random.default_rng(17)
    x = rng.standard_normal((8, C)).astype(np.float32)
    x[0] = 0.0                                                  # every group zero
    x[1, :G] = 0.0
    x[1, G:2 * G] = 1e30                                        # huge
    x[2] *= 1e-36                                               # subnormal-range groups
    x[3, :G] = np.float32(-0.01)
    x[3, 0] = np.float32(8.0)                                   # small negatives round to -0 / 0
    x[4, :G] = (np.arange(G) % 8 - 4).astype(np.float32) * 0.5  # exact grid points and ties
    x[5] *= 4000.0
    xb = wl.bf16_bits_from_f32(x)
    codes, scales = _run(bq, Tb, xb, fmt)
    y32 = wl.f32_from_bf16_bits(xb)                             # the identity transform is exact
    c_ref, s_ref = ob.quantize(y32, fmt)
    assert np.array_equal(scales, s_ref)
    assert np.array_equal(codes, c_ref)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_exact_rounding_ties(bq, fmt):
    """Identity blocks and groups whose scale is exact but whose reciprocal is not (0.375):
    every other value is a rounding tie of the format's grid (E2M1 midpoints for NVFP4,
    half-integers of the INT4 step), so the kernels' reciprocal products sit next to the
    boundary and must take IEEE division: codes bit-exact with the oracle."""
    G = ob.FORMATS[fmt]
    C = 256
    Tb = np.broadcast_to(wl.bf16_bits_from_f32(np.eye(G, dtype=np.float32)), (C // G, G, G)).copy()
    rng = np.random.default_rng(23)
    s = 0.375
    if fmt == "nvfp4":
        ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])   # E2M1 midpoints, in units of the scale
        amax = 6 * s                                             # scale = E4M3(amax / 6) = 0.375 exactly
    else:
        ties = np.arange(-7, 7) + 0.5                            # half-integers
        amax = 7 * s                                             # scale = fp16(amax / 7) = 0.375 exactly
    rows = []
    for r in range(6):
        v = s * rng.choice(ties, C) * rng.choice([-1.0, 1.0], C)
        v[::G] = amax * (1 if r % 2 else -1)                     # each group's absolute maximum
        v[1::2] = v[1::2] * (1 + 2.0 ** -7 * rng.choice([-1, 0, 1], C // 2))  # bf16 neighbours of ties
        rows.append(v)
    x = np.clip(np.stack(rows), -amax, amax).astype(np.float32)
    xb = wl.bf16_bits_from_f32(x)
    codes, scales = _run(bq, Tb, xb, fmt)
    y32 = wl.f32_from_bf16_bits(xb)                              # the identity transform is exact
    c_ref, s_ref = ob.quantize(y32, fmt)
    assert np.array_equal(scales, s_ref)
    assert np.array_equal(codes, c_ref)


@pytest.mark.parametrize("gscale", [2.0 ** -120, 1e-20, 3.0, 1e20, 2.0 ** 110])
def test_nvfp4_global_scale_extremes(bq, gscale):
    """Per-tensor scales that push den = s8 * gscale (or the quotients) out of the range
    where the reciprocal product is checked: those groups take IEEE division; codes and
    scales stay bit-exact with the oracle."""
    Tb, xb = _case(31, 64, 512, 16)
    codes, scales = _run(bq, Tb, xb, "nvfp4", gscale=gscale)
    y32 = _run(bq, Tb, xb, "none").astype(np.float32)
    c_ref, s_ref = ob.quantize(y32, "nvfp4", gscale)
    assert np.array_equal(scales, s_ref)
    assert np.array_equal(codes, c_ref)


def test_rejects_bad_shapes(bq):
    torch = H.torch()
    Tb, xb = _case(1, 4, 128, 32)
    bt = bq.BlockTransform(_dev_T(Tb))
    x = H.dev_bf16_bits(xb)
    codes, scales = bq.block_outputs(4, 128, "nvfp4", "cuda")
    with pytest.raises(bq.BQError):            # NVFP4 needs G = 16
        bq.bq_block_transform_quantize(bt, x, "nvfp4", codes, scales)
    with pytest.raises(ValueError):
        bq.BlockTransform(torch.zeros((2, 8, 8), dtype=torch.bfloat16, device="cuda"))
