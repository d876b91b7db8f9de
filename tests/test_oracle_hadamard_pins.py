"""Pins of the Hadamard preset in the oracle (oracle.butterfly.hadamard_preset_forward):
the library's Sylvester Hadamard matrix for the fixed preset, entries of magnitude
exactly 1/sqrt(n) and orthogonality for random quadrants, agreement with the general
butterfly at the same angles, and a planted mistake in the quadrant mapping."""

import numpy as np
import pytest

from oracle import butterfly as ob


def _dense(fn, n):
    return fn(np.eye(n)).T          # column j = Q e_j


@pytest.mark.parametrize("n", [2, 4, 8, 16, 64])
def test_fixed_preset_is_sylvester_hadamard_with_column_signs(n):
    scipy_linalg = pytest.importorskip("scipy.linalg")
    q = _dense(lambda x: ob.hadamard_preset_forward(None, x), n)
    d = np.array([1.0])
    for _ in range(int(np.log2(n))):
        d = np.kron(d, np.array([1.0, -1.0]))
    # Q = H_n diag(d) / sqrt(n), d the Kronecker power of (1, -1): the same identity
    # the general butterfly satisfies at theta = pi/4
    assert np.allclose(q, scipy_linalg.hadamard(n) * d[None, :] / np.sqrt(n), atol=1e-15)


@pytest.mark.parametrize("n,seed", [(8, 0), (16, 1), (128, 2)])
def test_random_quadrants_give_a_randomized_hadamard(n, seed):
    rng = np.random.default_rng(seed)
    L = int(np.log2(n))
    k = rng.integers(0, 4, size=(L, n // 2)).astype(np.uint8)
    q = _dense(lambda x: ob.hadamard_preset_forward(k, x), n)
    assert np.allclose(np.abs(q), 1.0 / np.sqrt(n), atol=1e-15)
    assert np.allclose(q @ q.T, np.eye(n), atol=1e-13)
    # the same transform as the general butterfly at theta = pi/4 + k pi/2 (whose
    # angles pass through float32, hence the 1e-7 tolerance)
    theta = (np.pi / 4 + k.astype(np.float64) * np.pi / 2).astype(np.float32)
    assert np.allclose(q, _dense(lambda x: ob.forward(theta, x), n), atol=1e-7)


def test_planted_quadrant_mapping_mistake_is_caught():
    n = 16
    rng = np.random.default_rng(7)
    k = rng.integers(0, 4, size=(4, n // 2)).astype(np.uint8)
    swapped = np.where(k == 1, 3, np.where(k == 3, 1, k)).astype(np.uint8)   # 3 pi/4 read as -pi/4
    theta = (np.pi / 4 + k.astype(np.float64) * np.pi / 2).astype(np.float32)
    good = _dense(lambda x: ob.forward(theta, x), n)
    bad = _dense(lambda x: ob.hadamard_preset_forward(swapped, x), n)
    assert np.abs(bad - good).max() > 0.1
