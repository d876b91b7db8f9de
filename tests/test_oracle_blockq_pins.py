"""Pins of the block-transform / block-quantizer oracle (oracle/blockq.py) against
independent constructions: a dense block-diagonal matrix, exact rational rounding,
brute-force searches, torch's FP8 E4M3 conversion, hand-worked fixtures and planted
mistakes."""

import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import blockq as ob

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_block_transform_is_block_diagonal_product():
    rng = np.random.default_rng(0)
    for G in (16, 32):
        T = rng.standard_normal((6, G, G))
        x = rng.standard_normal((5, 6 * G))
        D = scipy.linalg.block_diag(*T)                 # D[bG + o, bG + k] = T[b][o][k]
        assert np.allclose(ob.block_transform(T, x), x @ D.T, rtol=1e-13, atol=1e-13)


def test_planted_transposed_blocks_are_caught():
    rng = np.random.default_rng(1)
    T = rng.standard_normal((3, 16, 16))
    x = rng.standard_normal((2, 48))
    D = scipy.linalg.block_diag(*T)
    wrong = ob.block_transform(np.swapaxes(T, 1, 2), x)
    assert not np.allclose(wrong, x @ D.T)


def _e2m1_exact(v: Fraction):
    """Nearest E2M1 magnitude by exact rational arithmetic, ties to the even code."""
    grid = [Fraction(g).limit_denominator() for g in ob.E2M1_VALUES]
    a = abs(v)
    if a >= 6:
        return 7
    d = [abs(a - g) for g in grid]
    m = min(d)
    cands = [i for i, di in enumerate(d) if di == m]
    return cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]


def test_e2m1_rounding_matches_exact_rational_rounding():
    rng = np.random.default_rng(2)
    vals = np.concatenate([rng.uniform(-8, 8, 4000), np.arange(-70, 71) / 8.0,
                           np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.9, 1e6])])
    codes = ob.e2m1_code(vals)
    for v, c in zip(vals, codes):
        assert (c & 7) == _e2m1_exact(Fraction(float(v))), v
        assert bool(c & 8) == bool(np.signbit(v))


def test_planted_ties_to_odd_would_be_caught():
    # 1.25 sits between codes 2 (1.0) and 3 (1.5): the even code wins
    assert ob.e2m1_code(np.array([1.25]))[0] == 2
    assert ob.e2m1_code(np.array([1.75]))[0] == 4


def test_e4m3_rounding_and_bytes_match_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(50000) * 40, np.linspace(-448, 448, 9001),
                        2.0 ** np.arange(-9, 9), 3 * 2.0 ** np.arange(-9, 7), [0.0]])
    r = ob.e4m3_round(x.astype(np.float32))
    t = torch.tensor(x.astype(np.float32)).clamp(-448, 448).to(torch.float8_e4m3fn)
    assert np.array_equal(r, t.to(torch.float64).numpy())
    assert np.array_equal(ob.e4m3_bits(r), t.view(torch.uint8).numpy())
    assert ob.e4m3_round(np.array([1000.0, -1e9]))[0] == 448.0          # saturating
    assert ob.e4m3_round(np.array([1000.0, -1e9]))[1] == -448.0


def test_mxfp4_shared_exponent_per_binade():
    for k in range(-20, 20):
        for frac in (1.0, 1.3, 1.999):
            y = np.zeros((1, 32), np.float32)
            y[0, 5] = np.float32(frac * 2.0 ** k)
            _, sc = ob.quantize_mxfp4(y)
            assert int(sc[0, 0]) - 127 == k - 2
    _, sc = ob.quantize_mxfp4(np.zeros((1, 32), np.float32))
    assert sc[0, 0] == 0                                     # X = -127 for an all-zero group


def test_nvfp4_and_int4_against_brute_force():
    rng = np.random.default_rng(4)
    y = (rng.standard_normal((6, 64)) * rng.uniform(0.01, 30, (6, 1))).astype(np.float32)
    q, s8 = ob.quantize_nvfp4(y, gscale=0.75)
    for r in range(6):
        for g in range(4):
            den = np.float32(s8[r, g] * np.float32(0.75))
            for k in range(16):
                v = float(np.float32(y[r, 16 * g + k] / den))
                assert (q[r, 16 * g + k] & 7) == _e2m1_exact(Fraction(v))
    qi, s16 = ob.quantize_int4_sym(y)
    s = s16.view(np.float16).astype(np.float32)
    for r in range(6):
        for g in range(2):
            for k in range(32):
                v = Fraction(float(np.float32(y[r, 32 * g + k] / s[r, g])))
                best = min(range(-7, 8), key=lambda c: (abs(v - c), c % 2))
                assert qi[r, 32 * g + k] == best


def test_dequantized_error_bounds():
    """Every element within half a grid step of its value, except MXFP4 elements above 6
    units of the power-of-two scale (amax / 2^X lies in [4, 8)), which saturate to 6."""
    rng = np.random.default_rng(5)
    y = (rng.standard_normal((8, 256)) * 3).astype(np.float32)
    for fmt, G in (("mxfp4", 32), ("nvfp4", 16), ("int4", 32)):
        packed, sc = ob.quantize(y, fmt)
        d = ob.dequantize(packed, sc, fmt).reshape(8, -1, G)
        yv = y.reshape(8, -1, G).astype(np.float64)
        amax = np.abs(yv).max(-1)
        if fmt == "mxfp4":
            unit = 2.0 ** (sc.astype(np.float64) - 127)
            sat = np.abs(yv) > 6 * unit[..., None]
            # E2M1 steps: 0.5 up to 2, 1 up to 4, 2 up to 6 (units of the scale)
            half = np.where(np.abs(yv) <= 2 * unit[..., None], 0.25, np.where(np.abs(yv) <= 4 * unit[..., None], 0.5, 1.0))
            bound = np.where(sat, np.abs(yv) - 6 * unit[..., None], half * unit[..., None])
            assert np.all(np.abs(d - yv) <= bound + 1e-9)
            assert np.all(np.abs(yv) < 8 * unit[..., None])
        else:
            step = amax / 6.0 * 1.07 * 2.0 if fmt == "nvfp4" else amax / 7.0 * 1.001
            assert np.all(np.abs(d - yv).max(-1) <= step / 2 + 1e-6), fmt


@pytest.mark.parametrize("line", [l for l in open(os.path.join(GOLDEN, "blockq_handcases.txt"))
                                  if l.strip() and not l.startswith("#")])
def test_golden_handcases(line):
    fmt, vals, codes, scale = [p.strip() for p in line.split("|")]
    vals = np.array(vals.split(), dtype=np.float32)
    G = ob.FORMATS[fmt]
    y = np.zeros((1, G), np.float32)
    y[0, :len(vals)] = vals
    packed, sc = ob.quantize(y, fmt)
    q = ob.unpack4(packed)[0, :len(vals)]
    assert list(q) == [int(c) for c in codes.split()]
    assert int(np.asarray(sc).ravel()[0]) == int(scale)


def test_pack_layout():
    p = ob.pack4(np.array([[1, 2, 15, 0]], np.uint8))
    assert list(p[0]) == [0x21, 0x0F]
    assert list(ob.unpack4(ob.pack4(np.array([[-7, 7, -1, 3]], np.int8)), signed=True)[0]) == [-7, 7, -1, 3]
