"""Pins of the oracle quantizer: a hand-worked vector, the MSE of the scalar
stage on Gaussian coordinates, the pages' 0.983 cosine at 3 bits, the QJL
sign bits against an independent matrix product, and the zero vector."""
import numpy as np
import pytest
from scipy.linalg import hadamard

import oracle


def test_basis_vector_by_hand():
    # x = e_0: z = H D e_0 / 1 = delta_0 * (1, ..., 1); with b = 2 every z_j = +-1,
    # and 1 >= t_3 = (0.4528 + 1.5104)/2 -> code 3 for +1, code 0 for -1.
    d = 64
    k = oracle.make_constants(d, 2, 1)
    x = np.zeros((1, d))
    x[0, 0] = 1.0
    q = oracle.quantize(k, x)
    want_code = 3 if k.delta[0] > 0 else 0
    assert (q["codes"] == want_code).all()
    np.testing.assert_allclose(q["z"], k.delta[0] * np.ones((1, d)), rtol=0, atol=0)
    r = q["z"][0] - k.centroids[want_code]
    assert np.isclose(q["gamma"][0], np.sqrt(d) * abs(1 - k.centroids[3]), rtol=1e-14)
    np.testing.assert_array_equal(q["bits"][0], (k.S @ r >= 0).astype(np.uint8))


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_scalar_stage_mse_on_gaussian_coordinates(b):
    d = 128
    k = oracle.make_constants(d, b, 1)
    rng = np.random.default_rng(b)
    x = rng.standard_normal((2048, d))
    q = oracle.quantize(k, x, use_qjl=False)
    z = q["z"]
    zhat = k.centroids[q["codes"]]
    # z = H D x / ||x|| has unit-variance coordinates (||z||^2 = d exactly)
    np.testing.assert_allclose((z ** 2).sum(1), d, rtol=1e-12)
    err = ((z - zhat) ** 2).mean()
    # coordinates of a random direction: Beta law ~ N(0,1) up to O(1/d); 3 sigma + 2% model slack
    sig = ((z - zhat) ** 2).std() / np.sqrt(z.size)
    assert abs(err - k.mse) < 3 * sig + 0.02 * k.mse
    np.testing.assert_allclose(q["gamma"], np.sqrt(((z - zhat) ** 2).sum(1)), rtol=1e-12)
    np.testing.assert_allclose(q["norm"], np.linalg.norm(x, axis=1), rtol=1e-13)


def test_three_bit_cosine_matches_the_pages(golden_dir):
    want, tol = [float(v) for v in open(f"{golden_dir}/turboquant_cosine_3bit.txt").read().split("\n")[-2].split()]
    d = 128
    k = oracle.make_constants(d, 3, 1)
    x = np.random.default_rng(0).standard_normal((4096, d))
    q = oracle.quantize(k, x, use_qjl=False)
    zhat = k.centroids[q["codes"]]
    cos = (q["z"] * zhat).sum(1) / (np.linalg.norm(q["z"], axis=1) * np.linalg.norm(zhat, axis=1))
    assert abs(cos.mean() - want) <= tol
    assert abs(np.sqrt(1 - k.mse) - want) <= tol  # the closed form sqrt(1 - D_3) = 0.98257


def test_codes_count_thresholds_and_bits_match_matrix_products():
    d = 128
    k = oracle.make_constants(d, 2, 4)
    x = np.random.default_rng(3).standard_normal((64, d)) * 3 + 1
    q = oracle.quantize(k, x)
    z = (hadamard(d) @ (k.delta[:, None] * x.T)).T / np.linalg.norm(x, axis=1, keepdims=True)
    np.testing.assert_allclose(q["z"], z, rtol=1e-12, atol=1e-12)
    codes = (z[..., None] >= k.thresholds).sum(-1)
    np.testing.assert_array_equal(q["codes"], codes)
    r = z - k.centroids[codes]
    u = r @ k.S.T
    np.testing.assert_allclose(q["u"], u, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(q["bits"], (u >= 0).astype(np.uint8))


def test_zero_vector_gives_zero_record():
    k = oracle.make_constants(64, 3, 1)
    x = np.zeros((2, 64))
    x[1, 5] = -2.0
    q = oracle.quantize(k, x)
    assert (q["codes"][0] == 0).all() and (q["bits"][0] == 0).all()
    assert q["norm"][0] == 0 and q["gamma"][0] == 0
    assert q["norm"][1] == 2.0
