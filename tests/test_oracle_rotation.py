"""Pins for oracle.rotation: the randomized Walsh-Hadamard rotation.

[LP] 三.1: an orthogonal matrix preserves norms, H_n = H_1 (x) H_{n-1}; [LP] 二.2: y = H D x.
The independent references are scipy.linalg.hadamard (a library routine for the Sylvester
matrix) and the orthogonality identities.
"""
import numpy as np
import pytest
from scipy.linalg import hadamard

from oracle import rotation


@pytest.mark.parametrize("d", [1, 2, 4, 8, 16, 64, 128, 1024])
def test_fwht_matches_dense_hadamard(d):
    rng = np.random.default_rng(d)
    x = rng.standard_normal((5, d))
    H = hadamard(d).astype(np.float64)
    np.testing.assert_allclose(rotation.fwht(x), x @ H, rtol=0, atol=1e-10 * np.sqrt(d))


@pytest.mark.parametrize("d", [2, 8, 32, 256])
def test_sylvester_recursion_matches_library(d):
    np.testing.assert_array_equal(rotation.sylvester(d), hadamard(d))


@pytest.mark.parametrize("d", [8, 128])
def test_hadamard_is_scaled_orthogonal(d):
    H = rotation.sylvester(d)
    np.testing.assert_array_equal(H @ H.T, d * np.eye(d))


@pytest.mark.parametrize("d", [8, 128, 1024])
def test_rotation_preserves_norm_and_inverts(d):
    rng = np.random.default_rng(100 + d)
    D = rng.choice([-1.0, 1.0], size=d)
    u = rng.standard_normal((64, d))
    y = rotation.rotate(u, D)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(u, axis=1), rtol=1e-12)
    np.testing.assert_allclose(rotation.unrotate(y, D), u, rtol=0, atol=1e-12)


def test_rotation_equals_dense_form_d8():
    d = 8
    rng = np.random.default_rng(7)
    D = rng.choice([-1.0, 1.0], size=d)
    u = rng.standard_normal(d)
    dense = hadamard(d) @ np.diag(D) / np.sqrt(d)
    np.testing.assert_allclose(rotation.rotate(u[None], D)[0], dense @ u, atol=1e-14)


def test_rotation_spreads_an_outlier():
    # [JJ] 第二部分 第一步: after rotation no coordinate keeps the outlier's mass.
    d = 128
    D = np.random.default_rng(3).choice([-1.0, 1.0], size=d)
    e = np.zeros((1, d))
    e[0, 5] = 1.0
    y = rotation.rotate(e, D)
    np.testing.assert_allclose(np.abs(y), 1.0 / np.sqrt(d), rtol=1e-12)
