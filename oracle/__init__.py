"""CPU oracle for rotated-token KV-cache quantization (TurboQuant form).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg may import this package.  The
product library never loads it, and it shares no code, header, table or
constant generator with the CUDA path: the heavy loops live in
``oracle.cc`` (plain single-threaded fp64 C++), this module only marshals
numpy arrays and states the packed cache layout.

Parity status of every function here is pinned by ``tests/test_oracle_*.py``
(closed forms, textbook tables, published PRNG vectors, statistics and
brute force); nothing is "parity unpinned".

Packed cache layout (the pages give none; reading recorded in the design
notes).  Per stream of vectors (one (batch, head) of the cache, or one call
of the quantizer), for vector t:

* ``codes[t, p, w]`` (uint32): bit i = bit p of the Lloyd-Max code of
  coordinate 32*w + i, for planes p = 0..b-1 (bit-plane layout);
* ``qjl[t, w]`` (uint32): bit i = QJL sign bit of projection row 32*w + i;
* ``norms[t, 0:2]`` (fp16): (||x||, ||r||) -- for the NSN front end
  (||x||, ||w||);
* NSN only: ``block_mean[blk, j]`` (fp16), mean of block ``blk`` of 128
  tokens on channel j.

Block-32 layout (values): the same bits transposed per block of 32
consecutive vectors: ``codes[blk, p, j]`` bit i = bit p of the code of
coordinate j of vector 32*blk + i; ``qjl[blk, k]`` bit i = QJL bit of row k of
vector 32*blk + i; bits of vectors past the end are 0.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cc")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

NSN_BLOCK = 128


def build(force: bool = False) -> str:
    """Compile oracle.cc into liboracle.so next to it (g++, fp64, no fast-math)."""
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-o", tmp, _SRC])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            L.orc_splitmix64.restype = ctypes.c_uint64
            L.orc_splitmix64.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
            L.orc_rademacher_signs.argtypes = [ctypes.c_int, ctypes.c_uint64, P]
            L.orc_double_to_half.restype = ctypes.c_uint16
            L.orc_double_to_half.argtypes = [ctypes.c_double]
            L.orc_half_to_double.restype = ctypes.c_double
            L.orc_half_to_double.argtypes = [ctypes.c_uint16]
            L.orc_gaussian_fp16.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_uint64, P, P]
            L.orc_lloyd_max_gaussian.restype = ctypes.c_int
            L.orc_lloyd_max_gaussian.argtypes = [ctypes.c_int, P, P, P, ctypes.c_int, ctypes.c_double]
            L.orc_rht.argtypes = [ctypes.c_int, P, P, P]
            L.orc_qjl_sketch.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P, P]
            L.orc_qjl_estimate.restype = ctypes.c_double
            L.orc_qjl_estimate.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P, ctypes.c_double]
            L.orc_qjl_trials.argtypes = [ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int64, ctypes.c_uint64, P]
            L.orc_quantize.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P,
                                       P, ctypes.c_int64, P, P, P, P, P, P]
            L.orc_dequantize.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P,
                                         P, P, P, ctypes.c_int64, P]
            L.orc_decode_attend.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P,
                                            P, ctypes.c_int, P, P, P, P, P, P, P, P, ctypes.c_int64,
                                            ctypes.c_double, P, P]
            L.orc_nsn_quantize.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P,
                                           ctypes.c_int64, P, P, P, P, P, P, P]
            L.orc_nsn_dq_rec_bytes.restype = ctypes.c_int
            L.orc_nsn_dq_rec_bytes.argtypes = [ctypes.c_int, ctypes.c_int]
            L.orc_nsn_dq_quantize.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P, ctypes.c_int64,
                                              P, ctypes.c_int, P, P, P, P, P, P, P, P]
            _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ----------------------------------------------------------------------------
# Random numbers and number formats
# ----------------------------------------------------------------------------
def splitmix64(seed: int, i: int) -> int:
    return int(lib().orc_splitmix64(seed & (2**64 - 1), i))


def rademacher_signs(d: int, seed: int) -> np.ndarray:
    out = np.empty(d, np.int8)
    lib().orc_rademacher_signs(d, seed & (2**64 - 1), _p(out))
    return out


def gaussian_fp16(rows: int, cols: int, seed: int):
    """Returns (fp16 bit patterns uint16 [rows, cols], unrounded fp64 draws)."""
    bits = np.empty((rows, cols), np.uint16)
    draws = np.empty((rows, cols), np.float64)
    lib().orc_gaussian_fp16(rows, cols, seed & (2**64 - 1), _p(bits), _p(draws))
    return bits, draws


def double_to_half_bits(x) -> np.ndarray:
    x = np.asarray(x, np.float64)
    f = lib().orc_double_to_half
    return np.array([f(float(v)) for v in x.ravel()], np.uint16).reshape(x.shape)


def half_bits_to_double(h) -> np.ndarray:
    h = np.asarray(h, np.uint16)
    f = lib().orc_half_to_double
    return np.array([f(int(v)) for v in h.ravel()], np.float64).reshape(h.shape)


# ----------------------------------------------------------------------------
# Codebook and per-handle constants
# ----------------------------------------------------------------------------
def lloyd_max(b: int, max_iter: int = 1_000_000, tol: float = 1e-15):
    """Gaussian Lloyd-Max codebook: (centroids[2^b], thresholds[2^b-1], mse, steps)."""
    L = 1 << b
    c = np.empty(L, np.float64)
    t = np.empty(max(L - 1, 1), np.float64)
    mse = ctypes.c_double()
    it = lib().orc_lloyd_max_gaussian(b, _p(c), _p(t), ctypes.byref(mse), max_iter, tol)
    return c, t[: L - 1], mse.value, it


def sphere_coordinate_pdf(z, d: int):
    """Density of z = sqrt(d) u_1, u uniform on the unit sphere of R^d (d >= 3).

    TurboQuant blog, "Estágio 1": after the random rotation each coordinate of
    the unit vector follows Beta((d-1)/2, (d-1)/2) stretched to [-1, 1], i.e.
    f_u(u) = (1 - u^2)^((d-3)/2) / B(1/2, (d-1)/2); the quantizer works on
    z = sqrt(d) u (unit variance), so f(z) = f_u(z / sqrt(d)) / sqrt(d) on
    |z| < sqrt(d)."""
    from math import lgamma
    z = np.asarray(z, np.float64)
    a = (d - 3) / 2.0
    log_beta = lgamma(0.5) + lgamma((d - 1) / 2.0) - lgamma(d / 2.0)
    w = np.clip(1.0 - z * z / d, 0.0, None)
    return np.where(np.abs(z) < np.sqrt(d), w ** a, 0.0) / (np.exp(log_beta) * np.sqrt(d))


_GL = {}


def _cell_moments(d: int, lo: float, hi: float, nodes: int = 768):
    """int f, int z f, int z^2 f over [lo, hi] by Gauss-Legendre quadrature."""
    if nodes not in _GL:
        _GL[nodes] = np.polynomial.legendre.leggauss(nodes)
    x, w = _GL[nodes]
    z = 0.5 * (hi - lo) * x + 0.5 * (hi + lo)
    fw = 0.5 * (hi - lo) * w * sphere_coordinate_pdf(z, d)
    return fw.sum(), (fw * z).sum(), (fw * z * z).sum()


def lloyd_max_sphere(d: int, b: int, max_iter: int = 100_000, tol: float = 1e-14):
    """Lloyd-Max codebook for one coordinate of a rotated unit vector scaled by
    sqrt(d) (the d-exact law above instead of N(0, 1)): (centroids, thresholds,
    mse, steps).  Lloyd's two conditions, in the order the method states them:
    decision levels at the midpoints of adjacent centroids, each centroid the
    mean of its cell; iterated from the Gaussian codebook to a fixed point."""
    L = 1 << b
    edge = float(np.sqrt(d))
    c = lloyd_max(b)[0].copy()
    c *= min(1.0, 0.9 * edge / np.max(np.abs(c)))  # start inside the support, cells non-empty
    it = 0
    for it in range(1, max_iter + 1):
        t = np.concatenate(([-edge], 0.5 * (c[:-1] + c[1:]), [edge]))
        cn = np.empty(L)
        for k in range(L):
            p, m1, _ = _cell_moments(d, t[k], t[k + 1])
            cn[k] = m1 / p
        move = np.max(np.abs(cn - c))
        c = cn
        if move <= tol:
            break
    c = 0.5 * (c - c[::-1])  # the law is symmetric, so is the codebook
    t = np.concatenate(([-edge], 0.5 * (c[:-1] + c[1:]), [edge]))
    mse = 0.0
    for k in range(L):
        p, m1, m2 = _cell_moments(d, t[k], t[k + 1])
        mse += m2 - 2.0 * c[k] * m1 + c[k] * c[k] * p
    return c, t[1:-1].copy(), mse, it


@dataclass
class Constants:
    """Everything the method fixes for one (d, b, seed): signs, S, codebook.

    Reading of the pages (which give no PRNG): the Rademacher signs use the
    SplitMix64 stream seeded with ``seed``; the Gaussian projection S (m = d
    rows) uses the stream seeded with ``seed + 1`` and is rounded to fp16.
    """

    d: int
    b: int
    seed: int
    delta: np.ndarray          # int8 [d]
    S_half: np.ndarray         # uint16 [m, d] fp16 patterns
    S: np.ndarray              # float64 [m, d] (exact values of the fp16 entries)
    centroids: np.ndarray      # float64 [2^b]
    thresholds: np.ndarray     # float64 [2^b - 1]
    mse: float

    @property
    def m(self) -> int:
        return self.d


def make_constants(d: int, b: int, seed: int, codebook: str = "gaussian") -> Constants:
    """codebook: "gaussian" (Lloyd-Max for N(0, 1)) or "beta" (for the exact
    coordinate law of a rotated unit vector, lloyd_max_sphere)."""
    delta = rademacher_signs(d, seed)
    s_half, _ = gaussian_fp16(d, d, seed + 1)
    S = half_bits_to_double_fast(s_half)
    if codebook == "gaussian":
        c, t, mse, _ = lloyd_max(b)
    elif codebook == "beta":
        c, t, mse, _ = lloyd_max_sphere(d, b)
    else:
        raise ValueError(f"unknown codebook {codebook!r}")
    return Constants(d, b, seed, delta, s_half, S, c, t, mse)


def half_bits_to_double_fast(h) -> np.ndarray:
    """fp16 pattern -> value; via numpy's binary16 (exactly representable in fp64)."""
    return np.asarray(h, np.uint16).view(np.float16).astype(np.float64)


# ----------------------------------------------------------------------------
# The method
# ----------------------------------------------------------------------------
def rht(delta: np.ndarray, v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float64)
    d = v.shape[-1]
    y = np.empty(d, np.float64)
    lib().orc_rht(d, _p(_c(delta, np.int8)), _p(v), _p(y))
    return y


def qjl_sketch(S: np.ndarray, r: np.ndarray):
    S = _c(S, np.float64)
    r = _c(r, np.float64)
    m, d = S.shape
    bits = np.empty(m, np.uint8)
    u = np.empty(m, np.float64)
    lib().orc_qjl_sketch(m, d, _p(S), _p(r), _p(bits), _p(u))
    return bits, u


def qjl_estimate(S: np.ndarray, q: np.ndarray, bits: np.ndarray, rnorm: float) -> float:
    S = _c(S, np.float64)
    m, d = S.shape
    return float(lib().orc_qjl_estimate(m, d, _p(S), _p(_c(q, np.float64)), _p(_c(bits, np.uint8)),
                                        float(rnorm)))


def qjl_trials(m: int, q: np.ndarray, r: np.ndarray, T: int, seed0: int) -> np.ndarray:
    """T independent QJL estimates of <q, r>, each with its own fp16 Gaussian S (m x d)."""
    q = _c(q, np.float64)
    r = _c(r, np.float64)
    est = np.empty(T, np.float64)
    lib().orc_qjl_trials(m, q.shape[0], _p(q), _p(r), T, seed0 & (2**64 - 1), _p(est))
    return est


def quantize(k: Constants, x: np.ndarray, use_qjl: bool = True) -> dict:
    """Quantize rows of x ([n, d]) -> unpacked codes, bits, norms and intermediates."""
    x = _c(x, np.float64)
    n, d = x.shape
    assert d == k.d
    m = k.m if use_qjl else 0
    codes = np.empty((n, d), np.int32)
    bits = np.empty((n, max(m, 1)), np.uint8)
    norm = np.empty(n, np.float64)
    gamma = np.empty(n, np.float64)
    z = np.empty((n, d), np.float64)
    u = np.empty((n, max(m, 1)), np.float64)
    lib().orc_quantize(d, k.b, m, int(use_qjl), _p(k.delta), _p(k.S), _p(k.centroids), _p(k.thresholds),
                       _p(x), n, _p(codes), _p(bits), _p(norm), _p(gamma), _p(z), _p(u))
    out = dict(codes=codes, norm=norm, gamma=gamma, z=z)
    if use_qjl:
        out.update(bits=bits, u=u)
    return out


def dequantize(k: Constants, codes, bits, norm, gamma, use_qjl: bool = True) -> np.ndarray:
    codes = _c(codes, np.int32)
    n, d = codes.shape
    m = k.m if use_qjl else 0
    bits = _c(bits if use_qjl else np.zeros((n, 1)), np.uint8)
    xhat = np.empty((n, d), np.float64)
    lib().orc_dequantize(d, k.b, m, int(use_qjl), _p(k.delta), _p(k.S), _p(k.centroids), _p(codes), _p(bits),
                         _p(_c(norm, np.float64)), _p(_c(gamma, np.float64)), n, _p(xhat))
    return xhat


def decode_attend(k: Constants, q, kcache: dict, vcache: dict, scale: float, use_qjl: bool = True,
                  want_logits: bool = True):
    """Attention of G queries ([G, d]) over one KV head's key and value caches.

    Each cache is a dict with ``codes`` [T, d], ``bits`` [T, m] (when QJL is
    on), ``norm`` and ``gamma`` [T] -- the stored (fp16-widened) values.
    Returns (logits [G, T] or None, out [G, d]).
    """
    q = _c(np.atleast_2d(q), np.float64)
    G, d = q.shape
    m = k.m if use_qjl else 0

    def arrays(c):
        codes = _c(c["codes"], np.int32).reshape(-1, d)
        T = codes.shape[0]
        bits = _c(c["bits"] if use_qjl else np.zeros((max(T, 1), 1)), np.uint8)
        return codes, bits, _c(c["norm"], np.float64), _c(c["gamma"], np.float64), T

    kc, kb, kn, kg, T = arrays(kcache)
    vc, vb, vn, vg, Tv = arrays(vcache)
    assert T == Tv
    logits = np.empty((G, max(T, 1)), np.float64) if want_logits else None
    out = np.empty((G, d), np.float64)
    lib().orc_decode_attend(d, k.b, m, int(use_qjl), _p(k.delta), _p(k.S), _p(k.centroids), _p(q), G,
                            _p(kc), _p(kb), _p(kn), _p(kg), _p(vc), _p(vb), _p(vn), _p(vg), T,
                            float(scale), _p(logits), _p(out))
    return (logits[:, :T] if want_logits else None), out


def nsn_quantize(k: Constants, x, mean_in=None) -> dict:
    """NSN front end + quantizer (no QJL) on one head's tokens ([n_tok, d], n_tok % 128 == 0)."""
    x = _c(x, np.float64)
    n, d = x.shape
    assert n % NSN_BLOCK == 0
    nb = n // NSN_BLOCK
    codes = np.empty((n, d), np.int32)
    nx = np.empty(n, np.float64)
    nw = np.empty(n, np.float64)
    mean_half = np.empty((nb, d), np.uint16)
    mean_f64 = np.empty((nb, d), np.float64)
    z = np.empty((n, d), np.float64)
    mi = None if mean_in is None else _c(mean_in, np.uint16)
    lib().orc_nsn_quantize(d, k.b, NSN_BLOCK, _p(k.delta), _p(k.centroids), _p(k.thresholds), _p(x), n,
                           _p(mi), _p(codes), _p(nx), _p(nw), _p(mean_half), _p(mean_f64), _p(z))
    return dict(codes=codes, norm_x=nx, norm_w=nw, mean_half=mean_half, mean_f64=mean_f64, z=z)


def window_decode_attend(k: Constants, q, kcache: dict, vcache: dict, kwin, vwin, scale: float,
                         use_qjl: bool = True, nsn: tuple | None = None, dq: tuple | None = None):
    """Attention over a packed cache followed by a full-precision residual
    window (NSNQuant section 4: the newest tokens stay unquantized until a
    block is flushed).  The packed part is scored as in decode_attend (or
    nsn_decode_attend when ``nsn`` = (kmean, vmean), or nsn_dq_decode_attend
    when ``dq`` = (kside, vside)); the window's keys and values ([n_win, d],
    the stored fp16 values widened) are used exactly.  One softmax over all
    packed then window tokens.  Returns (logits over the packed then window
    tokens [G, T + n_win], out [G, d])."""
    q = _c(np.atleast_2d(q), np.float64)
    G, d = q.shape
    if dq is not None:
        lp, _ = nsn_dq_decode_attend(k, q, kcache, vcache, dq[0], dq[1], scale, want_logits=True)
        T = lp.shape[1]
        vh = nsn_dq_dequantize(k, vcache["codes"], vcache["norm_w"], dq[1])[:T] if T > 0 else np.zeros((0, d))
    elif nsn is None:
        lp, _ = decode_attend(k, q, kcache, vcache, scale, use_qjl, want_logits=True)
        T = lp.shape[1]
        vh = (dequantize(k, vcache["codes"], vcache.get("bits"), vcache["norm"], vcache["gamma"], use_qjl)
              if T > 0 else np.zeros((0, d)))
    else:
        lp, _ = nsn_decode_attend(k, q, kcache, vcache, nsn[0], nsn[1], scale, want_logits=True)
        T = lp.shape[1]
        vh = (nsn_dequantize(k, vcache["codes"], vcache["norm_x"], vcache["norm_w"], nsn[1])
              if T > 0 else np.zeros((0, d)))
    kw = np.asarray(kwin, np.float64).reshape(-1, d)
    vw = np.asarray(vwin, np.float64).reshape(-1, d)
    lw = scale * (q @ kw.T)
    logits = np.concatenate([lp, lw], axis=1)
    vals = np.concatenate([vh, vw], axis=0)
    if logits.shape[1] == 0:
        return logits, np.zeros((G, d))
    e = np.exp(logits - logits.max(axis=1, keepdims=True))
    return logits, (e @ vals) / e.sum(axis=1, keepdims=True)


def nsn_dequantize(k: Constants, codes, norm_x, norm_w, mean_half) -> np.ndarray:
    """Vectors stored by the NSN front end, reconstructed from its byproducts
    (NSNQuant section 1: x = s1 (s2 v + o) with s1 = ||x||/sqrt(d), s2 v = w):
    x_hat = ||x||/sqrt(d) (w_hat + o_blk), w_hat the plain dequantization of the
    codes with norm ||w|| (no QJL), o_blk the fp16 mean of the vector's block of
    128 tokens.  codes [n, d]; norm_x, norm_w [n]; mean_half [ceil(n/128), d] fp16 bits."""
    codes = _c(codes, np.int32)
    n, d = codes.shape
    w = dequantize(k, codes, None, norm_w, np.zeros(n), use_qjl=False)
    o = half_bits_to_double(np.asarray(mean_half, np.uint16).reshape(-1, d))
    o = np.repeat(o, NSN_BLOCK, axis=0)[:n]
    return (np.asarray(norm_x, np.float64) / np.sqrt(d))[:, None] * (w + o)


def nsn_decode_attend(k: Constants, q, kcache: dict, vcache: dict, kmean, vmean, scale: float,
                      want_logits: bool = True):
    """Attention of G queries ([G, d]) over NSN-stored keys and values of one
    KV head (NSNQuant section 4: attention from the byproducts).  Each cache is
    a dict with ``codes`` [T, d], ``norm_x`` and ``norm_w`` [T] (the stored
    fp16-widened values); kmean / vmean are the fp16 block means [ceil(T/128), d].
    Softmax in fp64 over the reconstructed vectors (nsn_dequantize)."""
    q = _c(np.atleast_2d(q), np.float64)
    Kh = nsn_dequantize(k, kcache["codes"], kcache["norm_x"], kcache["norm_w"], kmean)
    Vh = nsn_dequantize(k, vcache["codes"], vcache["norm_x"], vcache["norm_w"], vmean)
    G, d = q.shape
    if Kh.shape[0] == 0:
        return (np.zeros((G, 0)) if want_logits else None), np.zeros((G, d))
    logits = scale * (q @ Kh.T)
    e = np.exp(logits - logits.max(axis=1, keepdims=True))
    out = (e @ Vh) / e.sum(axis=1, keepdims=True)
    return (logits if want_logits else None), out


# ----------------------------------------------------------------------------
# NSN with double quantization of its side data (NSNQuant section 3)
# ----------------------------------------------------------------------------
def nsn_dq_rec_bytes(d: int, blk: int = NSN_BLOCK) -> int:
    """Bytes of one block's side record (see orc_nsn_dq_quantize)."""
    return int(lib().orc_nsn_dq_rec_bytes(d, blk))


def nsn_dq_quantize(k: Constants, x, side_in=None, blk: int = NSN_BLOCK, parts: int = 3) -> dict:
    """NSN front end with 4-bit norm and mean codes + the quantizer (no QJL) on one head's
    tokens ([n_tok, d], n_tok % blk == 0).  side_in (uint8 [n_tok/blk, rec_bytes]) replaces parts
    of the side records this function would write, which are then used as given: parts bit 0 the
    norm step and codes, bit 1 the mean offset, step and codes."""
    x = _c(x, np.float64)
    n, d = x.shape
    assert n % blk == 0
    nb = n // blk
    R = nsn_dq_rec_bytes(d, blk)
    codes = np.empty((n, d), np.int32)
    nw = np.empty(n, np.float64)
    side = np.empty((nb, R), np.uint8)
    n1 = np.empty(n, np.float64)
    oh = np.empty((nb, d), np.float64)
    of = np.empty((nb, d), np.float64)
    nx = np.empty(n, np.float64)
    z = np.empty((n, d), np.float64)
    si = None if side_in is None else _c(side_in, np.uint8).reshape(nb, R)
    lib().orc_nsn_dq_quantize(d, k.b, blk, _p(k.delta), _p(k.centroids), _p(k.thresholds), _p(x), n, _p(si),
                              int(parts), _p(codes), _p(nw), _p(side), _p(n1), _p(oh), _p(of), _p(nx), _p(z))
    return dict(codes=codes, norm_w=nw, side=side, n1=n1, o_hat=oh, mean_f64=of, norm_x=nx, z=z)


def nsn_dq_unpack(side, d: int, blk: int = NSN_BLOCK):
    """The stored scales and means of side records ([nb, rec_bytes] uint8), decoded as the
    format defines them: n1 = q nstep (exact), o_hat = fp32(lo + step q).  Returns
    (n1 [nb * blk], o_hat [nb, d]) in float64."""
    side = np.asarray(side, np.uint8).reshape(-1, nsn_dq_rec_bytes(d, blk))
    nb = side.shape[0]
    f16 = lambda lo, hi: (side[:, lo].astype(np.uint16) | (side[:, hi].astype(np.uint16) << 8)).view(np.float16)
    lo = f16(0, 1).astype(np.float64)
    st = f16(2, 3).astype(np.float64)
    ns = f16(4, 5).astype(np.float64)
    ob = side[:, 8:8 + d // 2]
    qo = np.stack([ob & 15, ob >> 4], axis=2).reshape(nb, d).astype(np.float64)
    nbt = side[:, 8 + d // 2:8 + d // 2 + blk // 2]
    qn = np.stack([nbt & 15, nbt >> 4], axis=2).reshape(nb, blk).astype(np.float64)
    o_hat = (lo[:, None] + st[:, None] * qo).astype(np.float32).astype(np.float64)
    n1 = (qn * ns[:, None]).reshape(-1)
    return n1, o_hat


def nsn_dq_dequantize(k: Constants, codes, norm_w, side, blk: int = NSN_BLOCK) -> np.ndarray:
    """Vectors stored with double-quantized side data: x_hat = n1/sqrt(d) (w_hat + o_hat)."""
    codes = _c(codes, np.int32)
    n, d = codes.shape
    n1, o_hat = nsn_dq_unpack(side, d, blk)
    w = dequantize(k, codes, None, norm_w, np.zeros(n), use_qjl=False)
    o = np.repeat(o_hat, blk, axis=0)[:n]
    return (n1[:n] / np.sqrt(d))[:, None] * (w + o)


def nsn_dq_decode_attend(k: Constants, q, kcache: dict, vcache: dict, kside, vside, scale: float,
                         want_logits: bool = True):
    """Attention of G queries over keys and values stored with double-quantized NSN side
    data; caches hold ``codes`` [T, d] and ``norm_w`` [T] (fp16-widened).  Softmax in fp64
    over the reconstructed vectors (nsn_dq_dequantize)."""
    q = _c(np.atleast_2d(q), np.float64)
    G, d = q.shape
    T = np.asarray(kcache["codes"]).reshape(-1, d).shape[0]
    if T == 0:
        return (np.zeros((G, 0)) if want_logits else None), np.zeros((G, d))
    Kh = nsn_dq_dequantize(k, kcache["codes"], kcache["norm_w"], kside)[:T]
    Vh = nsn_dq_dequantize(k, vcache["codes"], vcache["norm_w"], vside)[:T]
    logits = scale * (q @ Kh.T)
    e = np.exp(logits - logits.max(axis=1, keepdims=True))
    out = (e @ Vh) / e.sum(axis=1, keepdims=True)
    return (logits if want_logits else None), out


# ----------------------------------------------------------------------------
# Packed cache layout (see module docstring)
# ----------------------------------------------------------------------------
def pack_codes(codes: np.ndarray, b: int) -> np.ndarray:
    codes = np.asarray(codes, np.int64)
    n, d = codes.shape
    words = np.zeros((n, b, d // 32), np.uint32)
    for p in range(b):
        plane = ((codes >> p) & 1).astype(np.uint64).reshape(n, d // 32, 32)
        words[:, p, :] = (plane << np.arange(32, dtype=np.uint64)).sum(axis=2).astype(np.uint32)
    return words


def unpack_codes(words: np.ndarray, b: int, d: int) -> np.ndarray:
    words = np.asarray(words, np.uint32).reshape(-1, b, d // 32).astype(np.uint64)
    n = words.shape[0]
    codes = np.zeros((n, d), np.int32)
    sh = np.arange(32, dtype=np.uint64)
    for p in range(b):
        plane = ((words[:, p, :, None] >> sh) & 1).reshape(n, d).astype(np.int32)
        codes |= plane << p
    return codes


def pack_bits(bits: np.ndarray) -> np.ndarray:
    bits = np.asarray(bits, np.uint64)
    n, m = bits.shape
    return (bits.reshape(n, m // 32, 32) << np.arange(32, dtype=np.uint64)).sum(axis=2).astype(np.uint32)


def unpack_bits(words: np.ndarray, m: int) -> np.ndarray:
    words = np.asarray(words, np.uint32).reshape(-1, m // 32).astype(np.uint64)
    n = words.shape[0]
    return ((words[:, :, None] >> np.arange(32, dtype=np.uint64)) & 1).reshape(n, m).astype(np.uint8)


def pack_codes_block32(codes: np.ndarray, b: int) -> np.ndarray:
    codes = np.asarray(codes, np.int64)
    n, d = codes.shape
    nb = (n + 31) // 32
    full = np.zeros((nb * 32, d), np.int64)
    full[:n] = codes
    words = np.zeros((nb, b, d), np.uint32)
    sh = np.arange(32, dtype=np.uint64)[None, :, None]
    for p in range(b):
        plane = ((full >> p) & 1).astype(np.uint64).reshape(nb, 32, d)
        words[:, p, :] = (plane << sh).sum(axis=1).astype(np.uint32)
    return words


def unpack_codes_block32(words: np.ndarray, b: int, d: int, n: int) -> np.ndarray:
    words = np.asarray(words, np.uint32).reshape(-1, b, d).astype(np.uint64)
    nb = words.shape[0]
    codes = np.zeros((nb * 32, d), np.int32)
    sh = np.arange(32, dtype=np.uint64)[None, :, None]
    for p in range(b):
        plane = ((words[:, p, None, :] >> sh) & 1).reshape(nb * 32, d).astype(np.int32)
        codes |= plane << p
    return codes[:n]


def pack_bits_block32(bits: np.ndarray) -> np.ndarray:
    bits = np.asarray(bits, np.uint64)
    n, m = bits.shape
    nb = (n + 31) // 32
    full = np.zeros((nb * 32, m), np.uint64)
    full[:n] = bits
    return (full.reshape(nb, 32, m) << np.arange(32, dtype=np.uint64)[None, :, None]).sum(axis=1).astype(np.uint32)


def unpack_bits_block32(words: np.ndarray, m: int, n: int) -> np.ndarray:
    words = np.asarray(words, np.uint32).reshape(-1, m).astype(np.uint64)
    nb = words.shape[0]
    bits = ((words[:, None, :] >> np.arange(32, dtype=np.uint64)[None, :, None]) & 1).reshape(nb * 32, m)
    return bits[:n].astype(np.uint8)
