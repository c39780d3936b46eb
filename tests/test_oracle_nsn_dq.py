"""Pins of the NSN front end with double-quantized side data (NSNQuant summary,
section 3, "Double Quantization": the mean o and the scale s1 are stored with
4 bits, for about 0.23 bits per element of side data in all).

The format (a reading: the pages give none) is checked against what it must
satisfy independently of the code that writes it:
* the stored scale and mean are the ones the transform used, so the token is
  recovered exactly from them before its direction is coded;
* the 4-bit codes are within half a step of the values they stand for;
* zero tokens stay exactly zero;
* the byte count per element, which with the page's figure fixes the block;
* decode over such a cache is softmax attention over the reconstructed
  vectors, written out token by token with scipy's Hadamard matrix.
"""
import numpy as np
import pytest
from scipy.linalg import hadamard

import oracle
from calibration_free_rotated_token_b200 import workloads as wl


def _tokens(n, d, seed):
    return wl.nsn_tokens(1, n, d, seed=seed)[0].double().numpy()


@pytest.mark.parametrize("d,b", [(128, 2), (64, 1), (128, 3)])
def test_stored_scale_and_mean_recover_the_token(d, b):
    k = oracle.make_constants(d, b, 4)
    x = _tokens(256, d, 10 + d)
    r = oracle.nsn_dq_quantize(k, x)
    H = hadamard(d).astype(np.float64)
    # w from its codes' pre-image: z = H (delta .* w) / ||w||  =>  w = ||w||/d delta .* (H z)
    w = (r["norm_w"] / d)[:, None] * (k.delta[None, :] * (r["z"] @ H.T))
    o = np.repeat(r["o_hat"], 128, axis=0)
    xr = (r["n1"] / np.sqrt(d))[:, None] * (w + o)
    np.testing.assert_allclose(xr, x, rtol=1e-11, atol=1e-11 * np.abs(x).max())


def test_side_records_decode_to_the_values_used():
    d = 128
    k = oracle.make_constants(d, 2, 4)
    r = oracle.nsn_dq_quantize(k, _tokens(384, d, 3))
    n1, oh = oracle.nsn_dq_unpack(r["side"], d)
    np.testing.assert_array_equal(n1, r["n1"])
    np.testing.assert_array_equal(oh, r["o_hat"])
    # fp32 values: the mean is the sum of two fp16 numbers rounded once to fp32
    assert np.all(oh == oh.astype(np.float32).astype(np.float64))
    # re-running with the records as given reproduces everything
    r2 = oracle.nsn_dq_quantize(k, _tokens(384, d, 3), side_in=r["side"])
    for key in ("codes", "norm_w", "side", "n1", "o_hat"):
        np.testing.assert_array_equal(r2[key], r[key])


def test_codes_are_within_half_a_step():
    d = 128
    k = oracle.make_constants(d, 2, 4)
    x = _tokens(512, d, 5)
    r = oracle.nsn_dq_quantize(k, x)
    side = r["side"]
    f16 = lambda lo, hi: (side[:, lo].astype(np.uint16) | (side[:, hi].astype(np.uint16) << 8)).view(np.float16)
    lo, st, ns = (f16(0, 1).astype(np.float64), f16(2, 3).astype(np.float64), f16(4, 5).astype(np.float64))
    of = r["mean_f64"]
    # the mean codes cover [fp16(min), fp16(min) + 15 step] and every mean is within half a step
    # (plus the fp16 rounding of min and step)
    slack = 2.0 ** -11 * (np.abs(of).max(1) + 15 * st)
    assert np.all(np.abs(r["o_hat"] - of) <= 0.5 * st[:, None] + slack[:, None] + 1e-12)
    # norms: within half a step, except tiny ones which take the smallest nonzero code
    nx = r["norm_x"].reshape(-1, 128)
    n1 = r["n1"].reshape(-1, 128)
    big = nx >= 0.5 * ns[:, None]
    assert np.all(np.abs(n1 - nx)[big] <= 0.5 * np.broadcast_to(ns[:, None], nx.shape)[big] * (1 + 2.0 ** -10))
    assert np.all(n1[~big] == np.broadcast_to(ns[:, None], nx.shape)[~big])
    # max norm maps to 15 steps
    assert np.all(np.abs(n1.max(1) - nx.max(1)) <= 0.5 * ns * (1 + 2.0 ** -10) + 2.0 ** -11 * nx.max(1))


def test_zero_tokens_stay_zero():
    d = 64
    k = oracle.make_constants(d, 2, 4)
    x = _tokens(128, d, 6)
    x[[3, 77]] = 0.0
    r = oracle.nsn_dq_quantize(k, x)
    assert r["n1"][3] == 0 and r["n1"][77] == 0
    xh = oracle.nsn_dq_dequantize(k, r["codes"], r["norm_w"], r["side"])
    assert np.all(xh[[3, 77]] == 0)


def test_side_bytes_per_element_match_the_pages_figure_at_64_token_blocks():
    """fp16 ||w|| per token plus one side record per block.  With 128-token blocks (the NSN workload)
    the side data cost 0.195 bits per element at d = 128; with 64-token blocks the same format costs
    0.234, the pages' "about 0.23 bits"."""
    d = 128
    for blk, want in ((128, 0.1953125), (64, 0.234375)):
        R = oracle.nsn_dq_rec_bytes(d, blk)
        bits = (R + 2 * blk) * 8 / (blk * d)
        assert abs(bits - want) < 1e-12, (blk, bits)
    # without double quantization: fp16 ||x||, fp16 ||w|| per token and an fp16 mean per block
    assert (4 * 128 + 2 * d) * 8 / (128 * d) == 0.375


def test_decode_is_attention_over_tokens_rebuilt_one_by_one():
    d, T, G = 64, 256, 3
    k = oracle.make_constants(d, 2, 7)
    rk = oracle.nsn_dq_quantize(k, _tokens(T, d, 8))
    rv = oracle.nsn_dq_quantize(k, _tokens(T, d, 9))
    kc = dict(codes=rk["codes"], norm_w=rk["norm_w"].astype(np.float16).astype(np.float64))
    vc = dict(codes=rv["codes"], norm_w=rv["norm_w"].astype(np.float16).astype(np.float64))
    q = np.random.default_rng(1).standard_normal((G, d)) / 8
    l, o = oracle.nsn_dq_decode_attend(k, q, kc, vc, rk["side"], rv["side"], 0.7)
    H = hadamard(d).astype(np.float64)

    def rebuild(c, side):
        n1, oh = oracle.nsn_dq_unpack(side, d)
        out = np.empty((T, d))
        for t in range(T):
            w = c["norm_w"][t] / d * k.delta * (H @ k.centroids[c["codes"][t]])   # ||w||/d D H c[code]
            out[t] = n1[t] / np.sqrt(d) * (w + oh[t // 128])
        return out

    Kh, Vh = rebuild(kc, rk["side"]), rebuild(vc, rv["side"])
    lw = 0.7 * q @ Kh.T
    e = np.exp(lw - lw.max(1, keepdims=True))
    np.testing.assert_allclose(l, lw, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(o, (e @ Vh) / e.sum(1, keepdims=True), rtol=1e-10, atol=1e-12)


def test_double_quantization_keeps_the_reconstruction_quality():
    """On the NSN workload's distribution (off-centre channels, spread token norms) the coded tokens
    with 4-bit side data stay within 0.005 of the mean cosine that fp16 side data give, far above
    the plain quantizer without the front end."""
    d = 128
    k = oracle.make_constants(d, 2, 4)
    x = _tokens(1024, d, 11)
    r0 = oracle.nsn_quantize(k, x)
    x0 = oracle.nsn_dequantize(k, r0["codes"], r0["norm_x"], r0["norm_w"], r0["mean_half"])
    r1 = oracle.nsn_dq_quantize(k, x)
    x1 = oracle.nsn_dq_dequantize(k, r1["codes"], r1["norm_w"], r1["side"])
    cos = lambda a, b: ((a * b).sum(1) / np.linalg.norm(a, axis=1) / np.linalg.norm(b, axis=1)).mean()
    qp = oracle.quantize(k, x, False)
    xp = oracle.dequantize(k, qp["codes"], None, qp["norm"], qp["gamma"], False)
    c0, c1, cp = cos(x, x0), cos(x, x1), cos(x, xp)
    assert c1 > c0 - 0.005 and c1 > cp + 0.05, (c0, c1, cp)


def test_window_over_a_double_quantized_cache():
    """A double-quantized NSN cache followed by an exact window: with an empty window it is the cache's decode;
    in general one softmax over the tokens rebuilt from the stored values, then the window tokens."""
    d, T, W, G = 64, 256, 37, 2
    k = oracle.make_constants(d, 2, 12)
    rk = oracle.nsn_dq_quantize(k, _tokens(T, d, 21))
    rv = oracle.nsn_dq_quantize(k, _tokens(T, d, 22))
    kc = dict(codes=rk["codes"], norm_w=rk["norm_w"].astype(np.float16).astype(np.float64))
    vc = dict(codes=rv["codes"], norm_w=rv["norm_w"].astype(np.float16).astype(np.float64))
    rng = np.random.default_rng(3)
    q = rng.standard_normal((G, d)) / 8
    kw = rng.standard_normal((W, d)).astype(np.float16).astype(np.float64)
    vw = rng.standard_normal((W, d)).astype(np.float16).astype(np.float64)
    l0, o0 = oracle.window_decode_attend(k, q, kc, vc, np.zeros((0, d)), np.zeros((0, d)), 0.3, False,
                                         dq=(rk["side"], rv["side"]))
    l1, o1 = oracle.nsn_dq_decode_attend(k, q, kc, vc, rk["side"], rv["side"], 0.3)
    np.testing.assert_array_equal(l0, l1)
    np.testing.assert_allclose(o0, o1, rtol=1e-13, atol=1e-15)
    l, o = oracle.window_decode_attend(k, q, kc, vc, kw, vw, 0.3, False, dq=(rk["side"], rv["side"]))
    Kh = np.concatenate([oracle.nsn_dq_dequantize(k, kc["codes"], kc["norm_w"], rk["side"]), kw])
    Vh = np.concatenate([oracle.nsn_dq_dequantize(k, vc["codes"], vc["norm_w"], rv["side"]), vw])
    lw = 0.3 * q @ Kh.T
    e = np.exp(lw - lw.max(1, keepdims=True))
    np.testing.assert_allclose(l, lw, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o, (e @ Vh) / e.sum(1, keepdims=True), rtol=1e-11, atol=1e-13)
