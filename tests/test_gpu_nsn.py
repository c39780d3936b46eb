"""Parity of the CUDA NSN front end + quantizer with the CPU oracle.

The per-block channel mean is rounded to fp16 on both sides; the GPU
computes it in fp32, the oracle in fp64, so on a rounding tie the two may
pick the two neighbouring fp16 values.  Each GPU mean must equal the
oracle's rounding or, when the oracle's fp64 mean is within fp32 resolution
of the midpoint, the other neighbour; the oracle is then re-run with that
(oracle-derived) neighbour so that the codes are compared for the mean the
GPU actually subtracted."""
import numpy as np
import pytest
import torch

import oracle
from calibration_free_rotated_token_b200 import _abi as kvq
from calibration_free_rotated_token_b200 import workloads as wl

from .parity import CODE_BAND, max_excluded, to_np_f16bits, to_np_u32, ulp_distance_f16

pytestmark = pytest.mark.gpu


def run_nsn(h, x):
    H, T, d = x.shape
    codes = torch.empty((H, T, h.b, d // 32), dtype=torch.int32, device="cuda")
    norms = torch.empty((H, T, 2), dtype=torch.float16, device="cuda")
    means = torch.empty((H, T // 128, d), dtype=torch.float16, device="cuda")
    kvq.kvq_nsn_quantize(h, x, codes, norms, means)
    code, bits = kvq.kvq_status(h)
    assert code == 0, (code, bits)
    return codes, norms, means


def check_head(k, x, codes_g, norms_g, means_g):
    """x: [T, d] float64 of one head; GPU outputs of that head."""
    T, d = x.shape
    ref = oracle.nsn_quantize(k, x)
    mg = means_g.reshape(-1, d)
    mo = ref["mean_half"]
    differ = mg != mo
    stats = dict(mean_ties=int(differ.sum()))
    if differ.any():
        # the GPU's value must be the other fp16 neighbour of the fp64 mean, at a near-tie
        m64 = ref["mean_f64"][differ]
        r16 = mo[differ].view(np.float16)
        up = np.nextafter(r16, np.float16(np.inf))
        dn = np.nextafter(r16, np.float16(-np.inf))
        alt = np.where(r16.astype(np.float64) < m64, up, dn)
        assert np.array_equal(mg[differ].view(np.float16), alt), "block mean is not a neighbouring rounding"
        mid = 0.5 * (r16.astype(np.float64) + alt.astype(np.float64))
        assert np.all(np.abs(m64 - mid) <= 1e-6 * np.maximum(np.abs(m64), 1.0)), "mean rounding differs away from a tie"
        mean_in = mo.copy()
        mean_in[differ] = alt.view(np.uint16)
        ref = oracle.nsn_quantize(k, x, mean_in=mean_in)
    codes = oracle.unpack_codes(codes_g.reshape(T, -1), k.b, d)
    near = (np.abs(ref["z"][..., None] - k.thresholds) < CODE_BAND).any(-1)
    bad = (codes != ref["codes"]) & ~near
    assert bad.sum() == 0, f"{bad.sum()} codes differ outside the boundary band"
    assert near.sum() <= max_excluded(near.size), f"{near.sum()} excluded coordinates of {near.size}"
    nb = norms_g.reshape(T, 2)
    assert ulp_distance_f16(nb[:, 0], ref["norm_x"].astype(np.float16).view(np.uint16)).max() <= 1
    ok = ~near.any(1)
    assert ulp_distance_f16(nb[ok, 1], ref["norm_w"][ok].astype(np.float16).view(np.uint16)).max(initial=0) <= 1
    stats["excluded_coords"] = int(near.sum())
    return stats


@pytest.mark.parametrize("d,b,dtype", [(128, 2, torch.bfloat16), (128, 1, torch.float16), (64, 3, torch.float32),
                                       (64, 4, torch.bfloat16)])
def test_nsn_matches_oracle(d, b, dtype):
    x = wl.nsn_tokens(2, 512, d, seed=d + b, dtype=dtype)
    x[1, 130] = 0  # a zero token inside a block
    with kvq.Handle(d, b, 3, qjl=False) as h:
        codes, norms, means = run_nsn(h, x.cuda())
    k = oracle.make_constants(d, b, 3)
    for hh in range(2):
        check_head(k, x[hh].double().numpy(), to_np_u32(codes[hh]), to_np_f16bits(norms[hh]),
                   to_np_f16bits(means[hh]))


def test_nsn_rejects_ragged_tokens_and_qjl_handles():
    with kvq.Handle(128, 2, 3, qjl=False) as h:
        x = torch.randn(1, 200, 128, device="cuda", dtype=torch.bfloat16)
        with pytest.raises(kvq.KvqError):
            kvq.kvq_nsn_quantize(h, x, torch.empty(200 * 8, dtype=torch.int32, device="cuda"),
                                 torch.empty(400, dtype=torch.float16, device="cuda"),
                                 torch.empty(256, dtype=torch.float16, device="cuda"))
    with kvq.Handle(128, 2, 3, qjl=True) as h:
        x = torch.randn(1, 128, 128, device="cuda", dtype=torch.bfloat16)
        with pytest.raises(kvq.KvqError):
            kvq.kvq_nsn_quantize(h, x, torch.empty(128 * 8, dtype=torch.int32, device="cuda"),
                                 torch.empty(256, dtype=torch.float16, device="cuda"),
                                 torch.empty(128, dtype=torch.float16, device="cuda"))


def test_nsn_workload_full_size_sampled():
    """8 heads x 65536 tokens x 128 bf16, channel means N(0,3), token norms lognormal(0,0.7), b=2, no QJL."""
    c = wl.NSN
    x = wl.nsn_tokens(c["heads"], c["tokens"], c["d"], c["seed"], device="cuda")
    with kvq.Handle(c["d"], c["b"], c["handle_seed"], qjl=False) as h:
        codes, norms, means = run_nsn(h, x)
    k = oracle.make_constants(c["d"], c["b"], c["handle_seed"])
    rng = np.random.default_rng(4)
    for _ in range(3):
        hh = int(rng.integers(c["heads"]))
        blk = int(rng.integers(c["tokens"] // 128))
        sl = slice(blk * 128, (blk + 1) * 128)
        check_head(k, x[hh, sl].double().cpu().numpy(), to_np_u32(codes[hh, sl]), to_np_f16bits(norms[hh, sl]),
                   to_np_f16bits(means[hh, blk:blk + 1]))
    # the last block of the last head
    sl = slice(c["tokens"] - 128, c["tokens"])
    check_head(k, x[-1, sl].double().cpu().numpy(), to_np_u32(codes[-1, sl]), to_np_f16bits(norms[-1, sl]),
               to_np_f16bits(means[-1, -1:]))
