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


def _nsn_store(out):
    """What the NSN cache holds for a token: codes and the fp16-rounded (||x||, ||w||)."""
    return dict(codes=out["codes"], norm_x=out["norm_x"].astype(np.float16).astype(np.float64),
                norm_w=out["norm_w"].astype(np.float16).astype(np.float64))


def test_nsn_decode_reduces_to_plain_decode():
    """Zero block means and ||x|| = sqrt(d) (s1 = 1): the NSN reconstruction is the plain
    dequantization with norm ||w||, so NSN decode equals the plain decode (no QJL)."""
    d, T = 64, 300
    k = oracle.make_constants(d, 2, 3)
    rng = np.random.default_rng(6)
    st = []
    for _ in range(2):
        st.append(dict(codes=rng.integers(0, 4, (T, d)), norm_x=np.full(T, np.sqrt(d)),
                       norm_w=np.exp(rng.standard_normal(T))))
    zero = np.zeros((3, d), np.uint16)
    q = rng.standard_normal((2, d))
    ln, on = oracle.nsn_decode_attend(k, q, st[0], st[1], zero, zero, 0.3)
    plain = [dict(codes=s["codes"], norm=s["norm_w"], gamma=np.zeros(T)) for s in st]
    lp, op = oracle.decode_attend(k, q, plain[0], plain[1], 0.3, use_qjl=False)
    np.testing.assert_allclose(ln, lp, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(on, op, rtol=1e-12, atol=1e-12)


def test_nsn_decode_brute_force_tiny():
    """Explicit reconstruction x = ||x||/sqrt(d) (||w||/d delta .* (H c[code]) + o) with scipy's
    Sylvester matrix, then softmax attention written out token by token."""
    from scipy.linalg import hadamard
    d, T = 16, 200
    k = oracle.make_constants(d, 2, 4)
    rng = np.random.default_rng(7)
    H = hadamard(d).astype(np.float64)
    st = [dict(codes=rng.integers(0, 4, (T, d)), norm_x=np.exp(rng.standard_normal(T)),
               norm_w=np.exp(rng.standard_normal(T))) for _ in range(2)]
    means = [rng.standard_normal((2, d)).astype(np.float16).view(np.uint16) for _ in range(2)]
    q = rng.standard_normal((3, d))

    def rec(s, mh, t):
        o = mh.view(np.float16).astype(np.float64)[t // 128]
        w = s["norm_w"][t] / d * k.delta * (H @ k.centroids[s["codes"][t]])
        return s["norm_x"][t] / np.sqrt(d) * (w + o)

    Kx = np.array([rec(st[0], means[0], t) for t in range(T)])
    Vx = np.array([rec(st[1], means[1], t) for t in range(T)])
    for g in range(3):
        lg = np.array([0.5 * float(q[g] @ Kx[t]) for t in range(T)])
        wts = np.exp(lg - lg.max())
        og = sum(wts[t] * Vx[t] for t in range(T)) / wts.sum()
        ln, on = oracle.nsn_decode_attend(k, q[g], st[0], st[1], means[0], means[1], 0.5)
        np.testing.assert_allclose(ln[0], lg, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(on[0], og, rtol=1e-11, atol=1e-12)


def test_nsn_decode_tracks_exact_attention_on_shifted_data():
    """Tokens with per-channel means N(0, 3) and lognormal(0, 0.7) norms (the NSN workload's
    law), b = 2: attention over the NSN cache is close to exact fp64 attention, and far closer
    than over the plain quantizer's cache, which the channel means hurt (NSNQuant section 1)."""
    d, T = 128, 1024
    k = oracle.make_constants(d, 2, 1)
    rng = np.random.default_rng(8)
    mu = 3 * rng.standard_normal(d)
    K, V = [(rng.standard_normal((T, d)) + mu) * np.exp(0.7 * rng.standard_normal((T, 1))) for _ in range(2)]
    q = rng.standard_normal((4, d)) / np.sqrt(d)
    sc = 1 / np.sqrt(d)
    lx = sc * q @ K.T
    e = np.exp(lx - lx.max(1, keepdims=True))
    ox = (e @ V) / e.sum(1, keepdims=True)
    nk, nv = oracle.nsn_quantize(k, K), oracle.nsn_quantize(k, V)
    _, on = oracle.nsn_decode_attend(k, q, _nsn_store(nk), _nsn_store(nv), nk["mean_half"], nv["mean_half"], sc)
    pk, pv = oracle.quantize(k, K, False), oracle.quantize(k, V, False)
    plain = [dict(codes=p["codes"], norm=p["norm"].astype(np.float16).astype(np.float64), gamma=np.zeros(T))
             for p in (pk, pv)]
    _, op = oracle.decode_attend(k, q, plain[0], plain[1], sc, use_qjl=False)
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel(on, ox) < 0.02
    assert rel(op, ox) > 5 * rel(on, ox)
