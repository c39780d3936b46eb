"""NSN front end: the byproducts reconstruct the input (NSNQuant section 1),
the block mean is the per-channel mean of the normalized tokens, and the
quantized part equals the plain quantizer applied to the shifted tokens."""
import numpy as np

import oracle


def test_nsn_reconstruction_and_mean():
    d = 64
    k = oracle.make_constants(d, 2, 1)
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((256, d)) + 3 * rng.standard_normal(d)) * np.exp(0.7 * rng.standard_normal((256, 1)))
    out = oracle.nsn_quantize(k, x)
    u = np.sqrt(d) * x / np.linalg.norm(x, axis=1, keepdims=True)
    np.testing.assert_allclose(out["mean_f64"], u.reshape(2, 128, d).mean(1), rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(out["mean_half"], out["mean_f64"].astype(np.float16).view(np.uint16))
    o16 = np.repeat(out["mean_half"].view(np.float16).astype(np.float64), 128, axis=0)
    w = u - o16
    np.testing.assert_allclose(out["norm_w"], np.linalg.norm(w, axis=1), rtol=1e-13)
    # s1 (s2 v + o) = x with s1 = ||x||/sqrt d, s2 = ||w||/sqrt d, v = sqrt d w / ||w||
    s1 = out["norm_x"][:, None] / np.sqrt(d)
    s2 = out["norm_w"][:, None] / np.sqrt(d)
    v = np.sqrt(d) * w / out["norm_w"][:, None]
    np.testing.assert_allclose(s1 * (s2 * v + o16), x, rtol=1e-12, atol=1e-12)
    # the codes are the plain quantizer's codes of w
    q = oracle.quantize(k, w, use_qjl=False)
    np.testing.assert_array_equal(out["codes"], q["codes"])


def test_nsn_mean_override():
    d = 64
    k = oracle.make_constants(d, 2, 1)
    x = np.random.default_rng(5).standard_normal((128, d)) + 1.0
    out = oracle.nsn_quantize(k, x)
    alt = out["mean_half"].copy()
    alt[0, 3] += 1  # neighbouring fp16 value on channel 3
    out2 = oracle.nsn_quantize(k, x, mean_in=alt)
    np.testing.assert_array_equal(out2["mean_half"], alt)
    assert not np.allclose(out2["z"][:, :], out["z"][:, :], rtol=0, atol=0)
