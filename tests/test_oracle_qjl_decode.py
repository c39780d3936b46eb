"""The decode side of the QJL correction, tied to the pinned estimator.

TurboQuant blog, "Estagio 2: Correcao Residual QJL": the 1-bit sketch of the
residual corrects the inner product, and the corrected estimate is unbiased.
The estimator itself (``qjl_estimate``) is pinned by the 10^5-trial
unbiasedness test; these tests tie the coefficient that decode and
dequantization use to it:

* per key, the logit's QJL term is exactly the estimator's value on the
  rotated query and the stored residual norm;
* over independent Gaussian projections S (signs and codebook fixed), the
  decode logit, the decoded value and the dequantized key are unbiased for
  the exact inner products / vectors.  A QJL coefficient off by any constant
  factor (for instance sqrt(2/pi)/m in place of sqrt(pi/2)/m) moves the means
  by many standard errors.
"""
import numpy as np
import pytest

import oracle


def _stored(k, x, qjl=True, fp16_norms=True):
    q = oracle.quantize(k, x, qjl)
    n, g = q["norm"], q["gamma"]
    if fp16_norms:
        n = n.astype(np.float16).astype(np.float64)
        g = g.astype(np.float16).astype(np.float64)
    c = dict(codes=q["codes"], norm=n, gamma=g)
    if qjl:
        c["bits"] = q["bits"]
    return c


@pytest.mark.parametrize("d,b", [(64, 2), (128, 1), (128, 3), (256, 4)])
def test_logit_qjl_term_is_the_estimator(d, b):
    k = oracle.make_constants(d, b, 11)
    rng = np.random.default_rng(d * 10 + b)
    T = 40
    K = rng.standard_normal((T, d)) * 1.5 + 0.3
    kc = _stored(k, K)
    vc = _stored(k, rng.standard_normal((T, d)))
    q = rng.standard_normal(d)
    scale = 0.37
    logits, _ = oracle.decode_attend(k, q[None], kc, vc, scale, True)
    qr = oracle.rht(k.delta, q)                       # q' = H (delta .* q), pinned against scipy
    for t in range(T):
        code_term = qr @ k.centroids[kc["codes"][t]]
        est = oracle.qjl_estimate(k.S, qr, kc["bits"][t], kc["gamma"][t])
        want = scale * kc["norm"][t] / d * (code_term + est)
        assert np.isclose(logits[0, t], want, rtol=1e-12, atol=1e-13), t


def _constants_with_S(base, S_half):
    return oracle.Constants(base.d, base.b, base.seed, base.delta, S_half,
                            oracle.half_bits_to_double_fast(S_half), base.centroids, base.thresholds, base.mse)


def test_decode_unbiased_over_independent_projections():
    """Key logit, decoded value and dequantized key averaged over 12000 independent fp16 Gaussian S."""
    d, b, T = 32, 2, 12000
    base = oracle.make_constants(d, b, 21)
    rng = np.random.default_rng(5)
    x = rng.standard_normal(d) * 2.0
    v = rng.standard_normal(d)
    # queries along the vectors' residual directions make the QJL term large, so a wrong
    # coefficient shows; q2 probes the value
    q1 = x + 0.5 * rng.standard_normal(d)
    q2 = v + 0.5 * rng.standard_normal(d)
    scale = 0.5
    lg = np.empty(T)
    ov = np.empty(T)
    dk = np.empty(T)
    for i in range(T):
        s_half, _ = oracle.gaussian_fp16(d, d, 900_000 + i)
        k = _constants_with_S(base, s_half)
        kc = _stored(k, x[None], fp16_norms=False)
        vc = _stored(k, v[None], fp16_norms=False)
        l, o = oracle.decode_attend(k, q1[None], kc, vc, scale, True)
        lg[i] = l[0, 0]
        ov[i] = o[0] @ q2
        xh = oracle.dequantize(k, kc["codes"], kc["bits"], kc["norm"], kc["gamma"], True)
        dk[i] = xh[0] @ q1
    for est, truth, what in ((lg, scale * (q1 @ x), "logit"), (ov, q2 @ v, "decoded value"),
                             (dk, q1 @ x, "dequantized key")):
        se = est.std() / np.sqrt(T)
        assert abs(est.mean() - truth) < 4 * se, f"{what}: mean {est.mean()} vs {truth} (se {se})"
    # the code-only part is biased for these queries: without the correction the test would fail
    k0 = _constants_with_S(base, oracle.gaussian_fp16(d, d, 1)[0])
    xh0 = oracle.dequantize(k0, _stored(k0, x[None], False, False)["codes"], None,
                            np.array([np.linalg.norm(x)]), np.zeros(1), False)
    assert abs(xh0[0] @ q1 - q1 @ x) > 20 * dk.std() / np.sqrt(T)
