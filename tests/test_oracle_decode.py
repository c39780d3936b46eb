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


# ---------------------------------------------------------------------------
# packed cache + full-precision residual window
# ---------------------------------------------------------------------------
def _packed(k, X, qjl):
    q = oracle.quantize(k, X, qjl)
    st = dict(codes=q["codes"], norm=q["norm"].astype(np.float16).astype(np.float64),
              gamma=q["gamma"].astype(np.float16).astype(np.float64))
    if qjl:
        st["bits"] = q["bits"]
    return st


def test_window_decode_empty_window_is_packed_decode():
    d = 64
    k = oracle.make_constants(d, 2, 2)
    rng = np.random.default_rng(12)
    kst, vst = _packed(k, rng.standard_normal((300, d)), True), _packed(k, rng.standard_normal((300, d)), True)
    q = rng.standard_normal((2, d))
    lr, orf = oracle.decode_attend(k, q, kst, vst, 0.2, True)
    lw, ow = oracle.window_decode_attend(k, q, kst, vst, np.zeros((0, d)), np.zeros((0, d)), 0.2, True)
    np.testing.assert_allclose(lw, lr, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(ow, orf, rtol=1e-12, atol=1e-13)


def test_window_decode_only_window_is_exact_attention():
    d = 32
    k = oracle.make_constants(d, 1, 2)
    rng = np.random.default_rng(13)
    empty = dict(codes=np.zeros((0, d), np.int32), norm=np.zeros(0), gamma=np.zeros(0), bits=np.zeros((0, d)))
    Kw, Vw = rng.standard_normal((50, d)), rng.standard_normal((50, d))
    q = rng.standard_normal((3, d))
    lw, ow = oracle.window_decode_attend(k, q, empty, empty, Kw, Vw, 0.5, True)
    for g in range(3):
        l = np.array([0.5 * q[g] @ Kw[t] for t in range(50)])
        w = np.exp(l - l.max())
        np.testing.assert_allclose(lw[g], l, rtol=1e-13)
        np.testing.assert_allclose(ow[g], (w[:, None] * Vw).sum(0) / w.sum(), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("qjl", [True, False])
def test_window_decode_is_attention_over_reconstructed_then_window_tokens(qjl):
    """One softmax over the packed tokens (as reconstructed vectors, q . k_hat) followed by the
    window tokens, written out directly."""
    d, T, W = 64, 200, 37
    k = oracle.make_constants(d, 2, 3)
    rng = np.random.default_rng(14)
    K, V = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    kst, vst = _packed(k, K, qjl), _packed(k, V, qjl)
    Kh = oracle.dequantize(k, kst["codes"], kst.get("bits"), kst["norm"], kst["gamma"], qjl)
    Vh = oracle.dequantize(k, vst["codes"], vst.get("bits"), vst["norm"], vst["gamma"], qjl)
    Kw, Vw = rng.standard_normal((W, d)), rng.standard_normal((W, d))
    q = rng.standard_normal((2, d))
    lw, ow = oracle.window_decode_attend(k, q, kst, vst, Kw, Vw, 0.3, qjl)
    Kall, Vall = np.vstack([Kh, Kw]), np.vstack([Vh, Vw])
    l = 0.3 * q @ Kall.T
    e = np.exp(l - l.max(1, keepdims=True))
    np.testing.assert_allclose(lw, l, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(ow, (e @ Vall) / e.sum(1, keepdims=True), rtol=1e-10, atol=1e-11)
