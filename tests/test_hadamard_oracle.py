"""Pins for the Hadamard output projection in the oracle (no GPU).

The oracle builds H from the popcount definition; scipy.linalg.hadamard (a
library routine, Sylvester construction) pins it, and the algebraic properties
the page states (fixed orthogonal matrix, l2 norm preserved, an affine alpha /
beta rescaling after it) pin the projection."""
import numpy as np
import pytest
import scipy.linalg

import oracle


@pytest.mark.parametrize("n", [1, 2, 4, 8, 64, 1024])
def test_matrix_is_the_sylvester_hadamard_matrix(n):
    np.testing.assert_array_equal(oracle.hadamard_matrix(n) * np.sqrt(n), scipy.linalg.hadamard(n))


@pytest.mark.parametrize("n", [2, 16, 256])
def test_orthonormal_symmetric_involution(n):
    H = oracle.hadamard_matrix(n)
    np.testing.assert_allclose(H @ H.T, np.eye(n), atol=1e-12)
    np.testing.assert_array_equal(H, H.T)
    y = np.random.default_rng(0).standard_normal((5, n))
    z = oracle.hadamard_proj(y, np.ones(n), np.zeros(n))
    np.testing.assert_allclose(np.linalg.norm(z, axis=1), np.linalg.norm(y, axis=1), rtol=1e-12)
    np.testing.assert_allclose(oracle.hadamard_proj(z, np.ones(n), np.zeros(n)), y, atol=1e-12)


def test_small_cases_by_hand():
    # n = 2: H = [[1, 1], [1, -1]] / sqrt(2)
    z = oracle.hadamard_proj(np.array([[3.0, 1.0]]), np.array([2.0, 1.0]), np.array([0.5, -1.0]))
    np.testing.assert_allclose(z, [[2.0 * 4 / np.sqrt(2) + 0.5, 2 / np.sqrt(2) - 1.0]], atol=1e-14)
    # a unit vector e_0 maps to the constant row 1/sqrt(n)
    n = 8
    e0 = np.zeros((1, n))
    e0[0, 0] = 1.0
    np.testing.assert_allclose(oracle.hadamard_proj(e0, np.ones(n), np.zeros(n)), np.full((1, n), 1 / np.sqrt(8)))


def test_affine_part_is_elementwise():
    n = 32
    rng = np.random.default_rng(1)
    y = rng.standard_normal((3, n))
    a, b = rng.standard_normal(n), rng.standard_normal(n)
    base = oracle.hadamard_proj(y, np.ones(n), np.zeros(n))
    np.testing.assert_allclose(oracle.hadamard_proj(y, a, b), a * base + b, atol=1e-12)


def test_rejects_non_power_of_two():
    with pytest.raises(ValueError):
        oracle.hadamard_matrix(12)
