"""The oracle's Gaussian Lloyd-Max codebook against Max's table, the method's
stated MSE constants, closed forms and the fixed-point conditions by quadrature."""
import numpy as np
import pytest
from scipy import integrate, stats

import oracle


def _max_table(path):
    """{(levels, kind): [(value, one unit in its last printed digit), ...]}

    The 1960 table is accurate to about one unit in its last digit (e.g. the
    3-bit decision level 0.500550 is printed 0.5006)."""
    rows = {}
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            f = line.split()
            rows[(int(f[0]), f[1])] = [(float(v), 10.0 ** -len(v.split(".")[1])) for v in f[2:]]
    return rows


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_matches_max_table(b, golden_dir):
    tab = _max_table(f"{golden_dir}/lloyd_max_gaussian.txt")
    L = 1 << b
    c, t, mse, _ = oracle.lloyd_max(b)
    for got, (want, tol) in zip(c[L // 2:], tab[(L, "output")]):
        assert abs(got - want) <= tol
    if b > 1:
        for got, (want, tol) in zip(t[L // 2:], tab[(L, "decision")]):
            assert abs(got - want) <= tol
    # The 16-level MSE entry of the table (0.009497) sits 4e-6 below the value the
    # table's own levels give by quadrature (0.0095010, test_fixed_point_by_quadrature);
    # the MSE entries are therefore held to 1e-5, the levels to their printed digits.
    want, tol = tab[(L, "mse")][0]
    assert abs(mse - want) <= max(tol, 1e-5)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_stated_mse_constants(b, golden_dir):
    rows = [l.split() for l in open(f"{golden_dir}/lloyd_max_mse_target.txt") if l.strip() and not l.startswith("#")]
    target = {int(r[0]): (float(r[1]), float(r[2])) for r in rows}
    _, _, mse, _ = oracle.lloyd_max(b)
    want, tol = target[b]
    assert abs(mse - want) < tol


def test_one_bit_closed_form():
    c, t, mse, _ = oracle.lloyd_max(1)
    np.testing.assert_allclose(c, [-np.sqrt(2 / np.pi), np.sqrt(2 / np.pi)], rtol=1e-14)
    assert t[0] == 0.0
    assert abs(mse - (1 - 2 / np.pi)) < 1e-14


@pytest.mark.parametrize("b", [2, 3, 4])
def test_fixed_point_by_quadrature(b):
    c, t, mse, _ = oracle.lloyd_max(b)
    L = 1 << b
    np.testing.assert_allclose(c, -c[::-1], atol=1e-13)                      # symmetric
    np.testing.assert_allclose(t, 0.5 * (c[1:] + c[:-1]), rtol=0, atol=0)   # midpoints
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    D = 0.0
    for k in range(L):
        a, e = edges[k], edges[k + 1]
        p = integrate.quad(stats.norm.pdf, a, e, epsabs=1e-14, epsrel=1e-13)[0]
        m1 = integrate.quad(lambda x: x * stats.norm.pdf(x), a, e, epsabs=1e-14, epsrel=1e-13)[0]
        assert abs(m1 / p - c[k]) < 1e-9                                     # centroid = cell mean
        D += integrate.quad(lambda x: (x - c[k]) ** 2 * stats.norm.pdf(x), a, e, epsabs=1e-14,
                            epsrel=1e-13)[0]
    assert abs(D - mse) < 1e-10



# ---------------------------------------------------------------------------
# d-exact codebook: Lloyd-Max for one coordinate of a rotated unit vector,
# z = sqrt(d) u_1 with (u_1 + 1)/2 ~ Beta((d-1)/2, (d-1)/2).
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_sphere_codebook_d3_is_the_uniform_quantizer(b):
    """d = 3: u_1 is uniform on [-1, 1] (Archimedes), so z is uniform on
    [-sqrt(3), sqrt(3)] and Lloyd-Max is the uniform quantizer with MSE
    (cell width)^2 / 12 = 1 / L^2."""
    L = 1 << b
    c, t, mse, _ = oracle.lloyd_max_sphere(3, b)
    r = np.sqrt(3.0)
    np.testing.assert_allclose(c, r * (-1 + (2 * np.arange(L) + 1) / L), atol=1e-10)
    np.testing.assert_allclose(t, r * (-1 + 2 * np.arange(1, L) / L), atol=1e-10)
    assert abs(mse - 1.0 / L ** 2) < 1e-10


@pytest.mark.parametrize("d", [5, 64, 128, 256])
def test_sphere_codebook_one_bit_closed_form(d):
    """1 bit: the centroids are +-E|z| = sqrt(d) Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
    and the MSE is E[z^2] - E|z|^2 = 1 - E|z|^2."""
    from math import exp, lgamma, pi, sqrt
    e = sqrt(d) * exp(lgamma(d / 2) - lgamma((d + 1) / 2)) / sqrt(pi)
    c, t, mse, _ = oracle.lloyd_max_sphere(d, 1)
    np.testing.assert_allclose(c, [-e, e], rtol=1e-12)  # quadrature: ~1e-13 at d = 256
    assert t[0] == 0.0
    assert abs(mse - (1 - e * e)) < 1e-12


@pytest.mark.parametrize("d,b", [(64, 2), (128, 3), (256, 4), (64, 4)])
def test_sphere_codebook_against_scipy_beta(d, b):
    """Cell masses against scipy's Beta CDF and each centroid against the
    conditional mean integrated from scipy's Beta density (both independent of
    the oracle's density and quadrature); E[z^2] = MSE + sum_k P_k c_k^2 = 1."""
    a = (d - 1) / 2.0
    r = np.sqrt(d)
    law = stats.beta(a, a, loc=-r, scale=2 * r)  # z = sqrt(d) (2 B - 1)
    c, t, mse, _ = oracle.lloyd_max_sphere(d, b)
    edges = np.concatenate(([-r], t, [r]))
    P = np.diff(law.cdf(edges))
    assert abs(P.sum() - 1) < 1e-12
    for k in range(len(c)):
        lo, hi = edges[k], edges[k + 1]
        m1, _ = integrate.quad(lambda z: z * law.pdf(z), lo, hi, epsabs=1e-14, epsrel=1e-12, limit=200)
        assert abs(m1 / P[k] - c[k]) < 1e-9 * max(1.0, abs(c[k]))
    assert abs(mse + float(np.sum(P * c * c)) - 1.0) < 1e-11


def test_sphere_codebook_tends_to_the_gaussian_one():
    """u_1 sqrt(d) -> N(0, 1): the d-exact codebook approaches the Gaussian
    Lloyd-Max codebook, with an O(1/d) gap (4x smaller for 4x larger d)."""
    cg = oracle.lloyd_max(3)[0]
    gaps = [np.max(np.abs(oracle.lloyd_max_sphere(d, 3)[0] - cg)) for d in (512, 2048)]
    assert gaps[0] < 6e-3
    assert 3.0 < gaps[0] / gaps[1] < 5.0


def test_sphere_codebook_mse_on_random_unit_vectors():
    """Coordinates of uniformly random unit vectors (scaled by sqrt(d)): the
    d-exact codebook's empirical MSE matches its analytic MSE and is below the
    Gaussian codebook's on the same coordinates (it is optimal for that law)."""
    d, b, n = 64, 3, 40000
    rng = np.random.default_rng(11)
    g = rng.standard_normal((n, d))
    z = np.sqrt(d) * g / np.linalg.norm(g, axis=1, keepdims=True)
    cs, ts, mse_s, _ = oracle.lloyd_max_sphere(d, b)
    cg, tg, _, _ = oracle.lloyd_max(b)
    err_s = np.mean((z - cs[np.searchsorted(ts, z, side="right")]) ** 2)
    err_g = np.mean((z - cg[np.searchsorted(tg, z, side="right")]) ** 2)
    assert abs(err_s - mse_s) < 4e-4  # ~ 6 standard errors over n * d = 2.56e6 coordinates
    assert err_s < err_g
