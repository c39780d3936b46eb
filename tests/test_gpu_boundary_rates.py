"""Boundary-excluded code rate of each workload, pooled over a large sample.

The stated tolerance for codes: bit-exact except coordinates whose z lies
within 1e-5 of a decision level, and that count must stay below 1e-4 of all
coordinates.  Each test here quantizes one workload at full size on the GPU,
compares a large sample of it with the oracle (every call also checks the
adjacent-code rule), pools the excluded count over the whole sample and
checks the pooled rate against 1e-4 with no margin.  The counts are printed
in the terminal summary and, with KVQ_PARITY_RECORD=<path>, written there as
JSON.
"""
import concurrent.futures as cf
import os

import numpy as np
import pytest
import torch

import oracle
from calibration_free_rotated_token_b200 import _abi as kvq
from calibration_free_rotated_token_b200 import workloads as wl

from .parity import compare_quantize, oracle_quantize_threads, pooled_check, to_np_f16bits, to_np_u32

pytestmark = pytest.mark.gpu


def check_sample(k, X, codes, qjl, norms, use_qjl, pool, layout=0):
    ref = oracle_quantize_threads(k, X, use_qjl)
    return compare_quantize(k, X, codes, qjl, norms, use_qjl, ref=ref, layout=layout, pool=pool)


def sample_token_rows(k, Xg, codes, qjl, norms, use_qjl, rows, pool):
    ti = torch.from_numpy(rows).to(Xg.device)
    check_sample(k, Xg[ti].double().cpu().numpy(), to_np_u32(codes[ti]), to_np_u32(qjl[ti]) if use_qjl else None,
                 to_np_f16bits(norms[ti]), use_qjl, pool)


def sample_blocks(k, Xg, codes, qjl, norms, use_qjl, blocks, pool):
    """Whole blocks of 32 vectors of a block-32 output, gathered in order."""
    bi = torch.from_numpy(blocks).to(Xg.device)
    rows = (blocks[:, None] * 32 + np.arange(32)[None, :]).reshape(-1)
    ri = torch.from_numpy(rows).to(Xg.device)
    check_sample(k, Xg[ri].double().cpu().numpy(), to_np_u32(codes[bi]), to_np_u32(qjl[bi]) if use_qjl else None,
                 to_np_f16bits(norms[ri]), use_qjl, pool, layout=1)


def test_rate_tiny_reference():
    """All 4096 keys and 4096 values of the tiny workload (fp32 N(0,1), d 128, b 2 + QJL)."""
    c = wl.TINY
    k = oracle.make_constants(c["d"], c["b"], c["handle_seed"])
    with kvq.Handle(c["d"], c["b"], c["handle_seed"], qjl=True) as h:
        for seed, layout in ((c["data_seed"], 0), (c["data_seed"] + 1000, 1)):
            x = wl.gaussian(c["n"], c["d"], seed)
            codes, qj, norms = kvq.alloc_packed(h, c["n"], layout=layout)
            kvq.kvq_quantize(h, x.cuda(), codes, qj, norms, layout=layout)
            assert kvq.kvq_status(h)[0] == 0
            check_sample(k, x.double().numpy(), to_np_u32(codes), to_np_u32(qj), to_np_f16bits(norms), True,
                         "tiny_reference", layout=layout)
    print("tiny_reference", pooled_check("tiny_reference"))


def test_rate_llama_layer():
    """The layer's K and V (8 x 32768 x 128 bf16, b 2 + QJL) in one launch; 16384 key rows and
    512 value blocks (16384 vectors) sampled."""
    c = wl.LLAMA_LAYER
    k = oracle.make_constants(c["d"], c["b"], c["handle_seed"])
    K = wl.llama_keys(c["heads"], c["tokens"], c["d"], c["k_seed"], device="cuda").reshape(-1, c["d"])
    V = wl.llama_values(c["heads"], c["tokens"], c["d"], c["v_seed"], device="cuda").reshape(-1, c["d"])
    n = K.shape[0]
    rng = np.random.default_rng(10)
    with kvq.Handle(c["d"], c["b"], c["handle_seed"], qjl=True) as h:
        outK = kvq.alloc_packed(h, n)
        outV = kvq.alloc_packed(h, n, layout=1)
        kvq.kvq_quantize_batch(h, [(K, *outK, 0), (V, *outV, 1)])
        assert kvq.kvq_status(h)[0] == 0
        sample_token_rows(k, K, *outK, True, np.sort(rng.choice(n, 16384, replace=False)), "llama_layer")
        sample_blocks(k, V, *outV, True, np.sort(rng.choice(n // 32, 512, replace=False)), "llama_layer")
    print("llama_layer", pooled_check("llama_layer"))


def test_rate_decode_cache():
    """Keys and values of two (sequence, KV head) streams of the decode workload's cache
    (131072 tokens each, layer generator, b 2 + QJL); 16384 key rows and 512 value blocks."""
    c = wl.DECODE
    d, T = c["d"], c["T"]
    k = oracle.make_constants(d, c["b"], c["handle_seed"])
    rng = np.random.default_rng(11)
    with kvq.Handle(d, c["b"], c["handle_seed"], qjl=True) as h:
        for bi in (3, 12):
            K = wl.llama_keys(c["hkv"], T, d, wl.cache_slice_seed(c["handle_seed"], bi, 0, 0), device="cuda")[2]
            V = wl.llama_values(c["hkv"], T, d, wl.cache_slice_seed(c["handle_seed"], bi, 0, 1), device="cuda")[6]
            outK = kvq.alloc_packed(h, T)
            outV = kvq.alloc_packed(h, T, layout=1)
            kvq.kvq_quantize(h, K, *outK)
            kvq.kvq_quantize(h, V, *outV, layout=1)
            assert kvq.kvq_status(h)[0] == 0
            sample_token_rows(k, K, *outK, True, np.sort(rng.choice(T, 8192, replace=False)), "decode_cache")
            sample_blocks(k, V, *outV, True, np.sort(rng.choice(T // 32, 256, replace=False)), "decode_cache")
    print("decode_cache", pooled_check("decode_cache"))


def test_rate_nsn_front_end():
    """The NSN workload (8 x 65536 x 128 bf16, b 2): 160 sampled blocks of 128 tokens."""
    from .test_gpu_nsn import check_head, run_nsn

    c = wl.NSN
    x = wl.nsn_tokens(c["heads"], c["tokens"], c["d"], c["seed"], device="cuda")
    with kvq.Handle(c["d"], c["b"], c["handle_seed"], qjl=False) as h:
        codes, norms, means = run_nsn(h, x)
    k = oracle.make_constants(c["d"], c["b"], c["handle_seed"])
    rng = np.random.default_rng(12)
    picks = [(int(rng.integers(c["heads"])), int(rng.integers(c["tokens"] // 128))) for _ in range(160)]

    def one(p):
        hh, blk = p
        sl = slice(blk * 128, (blk + 1) * 128)
        return (x[hh, sl].double().cpu().numpy(), to_np_u32(codes[hh, sl]), to_np_f16bits(norms[hh, sl]),
                to_np_f16bits(means[hh, blk:blk + 1]))

    args = [one(p) for p in picks]
    with cf.ThreadPoolExecutor(max_workers=max(1, min(os.cpu_count() or 1, 32))) as ex:
        list(ex.map(lambda a: check_head(k, *a, pool="nsn_front_end"), args))
    print("nsn_front_end", pooled_check("nsn_front_end"))


def test_rate_sweep():
    """Every (d, b, QJL) of the sweep: 2^20 bf16 vectors (1% x10) quantized as keys; 4096 rows
    sampled per combination, pooled over the sweep (per-combination counts are printed)."""
    c = wl.SWEEP
    n = c["n"]
    per = {}
    for d in c["dims"]:
        x = wl.sweep_tokens(n, d, seed=c["seed"] + d, device="cuda")
        for b in c["bits"]:
            k = oracle.make_constants(d, b, c["handle_seed"])
            for qjl in c["qjl"]:
                with kvq.Handle(d, b, c["handle_seed"], qjl=qjl) as h:
                    codes, qj, norms = kvq.alloc_packed(h, n)
                    kvq.kvq_quantize(h, x, codes, qj, norms)
                    assert kvq.kvq_status(h)[0] == 0
                    rows = np.sort(np.random.default_rng(d * 100 + b * 10 + qjl).choice(n, 4096, replace=False))
                    ti = torch.from_numpy(rows).cuda()
                    st = check_sample(k, x[ti].double().cpu().numpy(), to_np_u32(codes[ti]),
                                      to_np_u32(qj[ti]) if qjl else None, to_np_f16bits(norms[ti]), qjl, "sweep")
                    per[f"d{d}_b{b}_{'qjl' if qjl else 'noqjl'}"] = (st["excluded_coords"], st["coords"])
    print("sweep per combination", per)
    print("sweep", pooled_check("sweep"))
