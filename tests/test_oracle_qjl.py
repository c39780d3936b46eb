"""The QJL estimator is unbiased over independent Gaussian projections
(TurboQuant blog, Stage 2: the 1-bit sketch removes the inner-product bias)."""
import numpy as np

import oracle


def test_qjl_estimator_unbiased_and_variance_bounded():
    d = m = 32
    rng = np.random.default_rng(7)
    q = rng.standard_normal(d)
    r = 0.3 * rng.standard_normal(d)
    T = 100_000
    est = oracle.qjl_trials(m, q, r, T, seed0=1000)
    truth = q @ r
    sd = est.std()
    assert abs(est.mean() - truth) < 4 * sd / np.sqrt(T)
    assert sd ** 2 <= np.pi / 2 * (q @ q) * (r @ r) / m


def test_qjl_estimate_consistent_with_sketch():
    d = m = 64
    k = oracle.make_constants(d, 2, 3)
    rng = np.random.default_rng(2)
    r = rng.standard_normal(d)
    q = rng.standard_normal(d)
    bits, u = oracle.qjl_sketch(k.S, r)
    np.testing.assert_allclose(u, k.S @ r, rtol=1e-12, atol=1e-12)
    est = oracle.qjl_estimate(k.S, q, bits, np.linalg.norm(r))
    want = np.sqrt(np.pi / 2) / m * np.linalg.norm(r) * ((k.S @ q) * (2.0 * bits - 1)).sum()
    assert np.isclose(est, want, rtol=1e-12)
