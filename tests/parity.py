"""Comparison rules between the CUDA path and the CPU oracle (test helper).

The tolerances are the method's stated ones:
* codes bit-exact, except coordinates whose oracle z lies within 1e-5 of a
  decision threshold; those are counted (must stay below 1e-4 of all
  coordinates) and must still hold one of the two codes adjacent to the
  threshold;
* QJL bits bit-exact except where |(S r)_i| < 1e-3 ||r||; vectors with an
  excluded code are left out of the bit and residual-norm checks;
* stored fp16 norms equal or one fp16 ulp apart (rounding-boundary cases),
  counted;
* logits and outputs |gpu - ref| <= 1e-4 + 2e-3 |ref| (fp32 accumulation).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

CODE_BAND = 1e-5
CODE_EXCL_MAX_FRAC = 1e-4

# Boundary-excluded coordinates pooled per workload.  The stated bar ("fewer
# than 1e-4 of all coordinates") is a rate: it is checked on the count pooled
# over every coordinate a workload's tests compare (pooled_check), not per
# call, where a few coordinates of noise on a small sample would decide it.
POOL: dict = {}
_POOL_LOCK = __import__("threading").Lock()


def pool_add(name: str, excluded: int, coords: int) -> None:
    with _POOL_LOCK:
        e = POOL.setdefault(name, [0, 0])
        e[0] += int(excluded)
        e[1] += int(coords)


def pooled(name: str) -> dict:
    ex, n = POOL.get(name, (0, 0))
    return {"excluded": ex, "coords": n, "rate": (ex / n) if n else 0.0}


def pooled_check(name: str) -> dict:
    """The pooled count of a workload against the stated rate, with no margin."""
    r = pooled(name)
    assert r["coords"] > 0, f"nothing pooled for {name}"
    assert r["excluded"] <= CODE_EXCL_MAX_FRAC * r["coords"], \
        f"{name}: {r['excluded']} boundary-excluded coordinates of {r['coords']} (rate {r['rate']:.2e} > 1e-4)"
    return r
QJL_BAND = 1e-3
ATOL, RTOL = 1e-4, 2e-3


def to_np_u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


def to_np_f16bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint16)


def ulp_distance_f16(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in fp16 ulps between non-negative fp16 patterns."""
    return np.abs(a_bits.astype(np.int64) - b_bits.astype(np.int64))


def compare_quantize(k: oracle.Constants, x: np.ndarray, codes_g, qjl_g, norms_g, use_qjl: bool,
                     ref: dict | None = None, layout: int = 0, pool: str | None = None) -> dict:
    """Checks one quantize call (layout 0: one record per vector, 1: block-32); returns counts.
    The boundary-excluded count is added to the workload `pool` (checked by pooled_check)."""
    x = np.asarray(x, np.float64)
    n, d = x.shape
    if ref is None:
        ref = oracle.quantize(k, x, use_qjl)
    if layout == 0:
        codes = oracle.unpack_codes(codes_g.reshape(n, -1), k.b, d)
    else:
        codes = oracle.unpack_codes_block32(codes_g, k.b, d, n)
    near = (np.abs(ref["z"][..., None] - k.thresholds[None, None, :]) < CODE_BAND).any(-1)
    near[ref["norm"] == 0] = False  # a zero vector has a defined all-zero record: compared exactly
    bad = (codes != ref["codes"]) & ~near
    assert bad.sum() == 0, f"{bad.sum()} codes differ outside the boundary band (first at {np.argwhere(bad)[:5]})"
    if pool is not None:
        pool_add(pool, near.sum(), near.size)
    # excluded coordinates must hold one of the two codes adjacent to a nearby threshold
    if near.any():
        zc = ref["z"][near]
        kk = np.argmin(np.abs(zc[:, None] - k.thresholds[None, :]), axis=1)
        got = codes[near]
        assert np.all((got == kk) | (got == kk + 1)), "an excluded coordinate holds a non-adjacent code"
    vec_ok = ~near.any(1)
    norm_bits = norms_g.reshape(n, 2)
    want_n = ref["norm"].astype(np.float16).view(np.uint16)
    dn = ulp_distance_f16(norm_bits[:, 0], want_n)
    assert dn.max(initial=0) <= 1, f"norm off by {dn.max()} ulp"
    want_g = ref["gamma"].astype(np.float16).view(np.uint16)
    dg = ulp_distance_f16(norm_bits[:, 1], want_g)[vec_ok]
    assert dg.max(initial=0) <= 1, f"gamma off by {dg.max()} ulp"
    out = dict(excluded_coords=int(near.sum()), coords=int(near.size), norm_ulp=int((dn > 0).sum()),
               gamma_ulp=int((dg > 0).sum()))
    if use_qjl:
        bits = oracle.unpack_bits(qjl_g.reshape(n, -1), k.m) if layout == 0 else oracle.unpack_bits_block32(qjl_g, k.m, n)
        tiny = np.abs(ref["u"]) < QJL_BAND * ref["gamma"][:, None]
        cmp = ~tiny & vec_ok[:, None]
        badb = (bits != ref["bits"]) & cmp
        assert badb.sum() == 0, f"{badb.sum()} QJL bits differ outside the band (first at {np.argwhere(badb)[:5]})"
        out["excluded_bits"] = int((~cmp).sum())
    return out


def assert_close(got: np.ndarray, want: np.ndarray, what: str):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    finite = np.isfinite(want)
    assert np.array_equal(np.isfinite(got), finite), f"{what}: non-finite pattern differs"
    err = np.abs(got[finite] - want[finite])
    lim = ATOL + RTOL * np.abs(want[finite])
    worst = np.max(err / lim, initial=0.0)
    assert worst <= 1.0, f"{what}: max |err| / (1e-4 + 2e-3 |ref|) = {worst:.3f}"
    return worst


def oracle_quantize_threads(k: oracle.Constants, x: np.ndarray, use_qjl: bool) -> dict:
    """oracle.quantize of the rows of x, over row ranges on the host cores (the C oracle runs
    without the interpreter lock; the ranges share nothing), concatenated in order."""
    import concurrent.futures as cf
    import os

    x = np.asarray(x, np.float64)
    parts = [p for p in np.array_split(x, max(1, min(os.cpu_count() or 1, 32))) if p.shape[0]]
    if len(parts) <= 1:
        return oracle.quantize(k, x, use_qjl)
    with cf.ThreadPoolExecutor(max_workers=len(parts)) as ex:
        outs = list(ex.map(lambda p: oracle.quantize(k, p, use_qjl), parts))
    return {key: np.concatenate([o[key] for o in outs]) for key in outs[0]}


def oracle_cache(k: oracle.Constants, x: np.ndarray, use_qjl: bool, layout: int = 0):
    """The oracle's own packed cache of x: (codes u32, qjl u32 or None, norms fp16, widened dict)."""
    q = oracle_quantize_threads(k, x, use_qjl)
    if layout == 0:
        codes = oracle.pack_codes(q["codes"], k.b)
        qjl = oracle.pack_bits(q["bits"]) if use_qjl else None
    else:
        codes = oracle.pack_codes_block32(q["codes"], k.b)
        qjl = oracle.pack_bits_block32(q["bits"]) if use_qjl else None
    nb = q["norm"].astype(np.float16)
    gb = q["gamma"].astype(np.float16)
    norms = np.stack([nb, gb], axis=1)
    stored = dict(codes=q["codes"], norm=nb.astype(np.float64), gamma=gb.astype(np.float64))
    if use_qjl:
        stored["bits"] = q["bits"]
    return codes, qjl, norms, stored


def to_device_u32(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(device)
