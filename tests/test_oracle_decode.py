"""Decode attention from the rotated domain against brute-force attention
over explicitly dequantized vectors (inverse rotation, PolarQuant
"Dequantizacao"), in fp64, on tiny inputs."""
import numpy as np
import pytest

import oracle


def _softmax_attend(q, keys, vals, scale):
    l = scale * q @ keys.T
    w = np.exp(l - l.max(axis=1, keepdims=True))
    return l, (w @ vals) / w.sum(axis=1, keepdims=True)


def _stored(k, x, qjl):
    """Quantize and keep what the cache stores (fp16 norms)."""
    q = oracle.quantize(k, x, qjl)
    c = dict(codes=q["codes"], norm=q["norm"].astype(np.float16).astype(np.float64),
             gamma=q["gamma"].astype(np.float16).astype(np.float64))
    if qjl:
        c["bits"] = q["bits"]
    return c


@pytest.mark.parametrize("d,b,qjl", [(64, 2, True), (128, 3, True), (64, 1, False), (128, 4, False)])
def test_rotated_domain_equals_dequantized_attention(d, b, qjl):
    k = oracle.make_constants(d, b, 5)
    rng = np.random.default_rng(d + b)
    T, G = 48, 4
    kc = _stored(k, rng.standard_normal((T, d)) * 2 + 0.5, qjl)
    vc = _stored(k, rng.standard_normal((T, d)), qjl)
    q = rng.standard_normal((G, d))
    Kh = oracle.dequantize(k, kc["codes"], kc.get("bits"), kc["norm"], kc["gamma"], qjl)
    Vh = oracle.dequantize(k, vc["codes"], vc.get("bits"), vc["norm"], vc["gamma"], qjl)
    scale = 1 / np.sqrt(d)
    l_ref, o_ref = _softmax_attend(q, Kh, Vh, scale)
    l, o = oracle.decode_attend(k, q, kc, vc, scale, qjl)
    np.testing.assert_allclose(l, l_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)


def test_dequantized_reconstruction_error_matches_mse():
    d = 128
    k = oracle.make_constants(d, 3, 2)
    x = np.random.default_rng(0).standard_normal((512, d))
    qx = oracle.quantize(k, x, use_qjl=False)
    xh = oracle.dequantize(k, qx["codes"], None, qx["norm"], qx["gamma"], use_qjl=False)
    # rotation is an isometry up to sqrt(d): ||x - xhat||^2 / ||x||^2 = ||z - zhat||^2 / d
    rel = ((x - xh) ** 2).sum(1) / (x ** 2).sum(1)
    np.testing.assert_allclose(rel, qx["gamma"] ** 2 / d, rtol=1e-10)


def test_qjl_term_reduces_logit_error():
    # the residual sketch should make <q, khat> closer to <q, k> on average (TurboQuant Stage 2)
    d = 128
    k = oracle.make_constants(d, 2, 3)
    rng = np.random.default_rng(9)
    K = rng.standard_normal((512, d))
    q = rng.standard_normal((1, d))
    with_q = _stored(k, K, True)
    Kh1 = oracle.dequantize(k, with_q["codes"], with_q["bits"], with_q["norm"], with_q["gamma"], True)
    Kh0 = oracle.dequantize(k, with_q["codes"], None, with_q["norm"], with_q["gamma"], False)
    e1 = ((q @ (Kh1 - K).T) ** 2).mean()
    e0 = ((q @ (Kh0 - K).T) ** 2).mean()
    bias0 = (q @ (Kh0 - K).T).mean()
    assert e1 < e0 * 1.5 and abs((q @ (Kh1 - K).T).mean()) <= abs(bias0) + 3 * np.sqrt(e1 / 512)


def test_empty_context_gives_zero_output():
    k = oracle.make_constants(64, 2, 1)
    empty = dict(codes=np.zeros((0, 64), np.int32), bits=np.zeros((0, 64), np.uint8), norm=np.zeros(0),
                 gamma=np.zeros(0))
    _, o = oracle.decode_attend(k, np.ones((2, 64)), empty, empty, 1.0, True)
    assert (o == 0).all()
