"""The oracle's randomized Hadamard rotation against the textbook Sylvester matrix."""
import numpy as np
import pytest
from scipy.linalg import hadamard

import oracle


@pytest.mark.parametrize("d", [64, 128, 256])
def test_rht_equals_sylvester_matrix_product(d):
    rng = np.random.default_rng(d)
    delta = oracle.rademacher_signs(d, 9)
    x = rng.standard_normal(d)
    np.testing.assert_allclose(oracle.rht(delta, x), hadamard(d) @ (delta * x), rtol=1e-13, atol=1e-12)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_rht_orthogonality_and_self_inverse(d):
    ones = np.ones(d, np.int8)
    H = np.stack([oracle.rht(ones, e) for e in np.eye(d)], axis=1)  # columns H e_j
    np.testing.assert_array_equal(H @ H.T, d * np.eye(d))          # H H^T = d I (integers)
    np.testing.assert_array_equal(H, H.T)                           # symmetric => H H = d I
    rng = np.random.default_rng(1)
    delta = oracle.rademacher_signs(d, 3)
    x = rng.standard_normal(d)
    y = oracle.rht(delta, x)
    assert np.isclose(y @ y, d * (x @ x), rtol=1e-13)               # ||H D x||^2 = d ||x||^2
    back = delta * oracle.rht(ones, y) / d                           # D H (H D x) / d = x
    np.testing.assert_allclose(back, x, rtol=1e-12, atol=1e-12)
