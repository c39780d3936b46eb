"""Parity of the CUDA quantizer (through the C ABI) with the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from calibration_free_rotated_token_b200 import _abi as kvq
from calibration_free_rotated_token_b200 import workloads as wl

from .parity import compare_quantize, to_np_f16bits, to_np_u32

pytestmark = pytest.mark.gpu

_consts = {}


def constants(d, b, seed):
    key = (d, b, seed)
    if key not in _consts:
        _consts[key] = oracle.make_constants(d, b, seed)
    return _consts[key]


def run_quantize(h, x, layout=0):
    codes, qjl, norms = kvq.alloc_packed(h, x.shape[0], layout=layout)
    kvq.kvq_quantize(h, x, codes, qjl, norms, layout=layout)
    code, bits = kvq.kvq_status(h)
    assert code == 0, (code, bits, kvq.kvq_last_error())
    return codes, qjl, norms


@pytest.mark.parametrize("d,b", [(64, 1), (128, 2), (256, 3), (128, 4)])
def test_constants_match_oracle(d, b):
    with kvq.Handle(d, b, 7, qjl=True) as h:
        signs, S, cent, thr = kvq.kvq_get_constants(h)
    k = constants(d, b, 7)
    np.testing.assert_array_equal(signs.numpy(), k.delta)
    np.testing.assert_array_equal(S.numpy().view(np.uint16), k.S_half)
    # two independent Lloyd-Max computations: equal to fp32 rounding
    np.testing.assert_allclose(cent.numpy(), k.centroids, rtol=2.0 ** -23, atol=1e-12)
    np.testing.assert_allclose(thr.numpy(), k.thresholds, rtol=2.0 ** -23, atol=1e-12)


def test_tiny_reference_workload():
    """4096 fp32 N(0,1) keys, d=128, b=2 + QJL (m=128), data seed 0, signs seed 1, S seed 2."""
    c = wl.TINY
    x = wl.gaussian(c["n"], c["d"], c["data_seed"])
    with kvq.Handle(c["d"], c["b"], c["handle_seed"], qjl=True) as h:
        codes, qjl, norms = run_quantize(h, x.cuda())
    k = constants(c["d"], c["b"], c["handle_seed"])
    stats = compare_quantize(k, x.double().numpy(), to_np_u32(codes), to_np_u32(qjl), to_np_f16bits(norms), True)
    print("tiny:", stats)


CASES = [
    # d, b, qjl, dtype, n  (n spans several tiles and a ragged tail)
    (128, 2, True, torch.bfloat16, 1000),
    (128, 2, False, torch.bfloat16, 777),
    (128, 1, True, torch.float16, 515),
    (128, 3, True, torch.float32, 300),
    (128, 4, False, torch.bfloat16, 640),
    (64, 1, True, torch.bfloat16, 1000),
    (64, 2, True, torch.float32, 333),
    (64, 3, False, torch.float16, 257),
    (64, 4, True, torch.bfloat16, 129),
    (256, 1, True, torch.bfloat16, 300),
    (256, 2, True, torch.float16, 1000),
    (256, 3, False, torch.bfloat16, 450),
    (256, 4, True, torch.bfloat16, 129),
]


@pytest.mark.parametrize("d,b,qjl,dtype,n", CASES)
def test_quantize_matches_oracle(d, b, qjl, dtype, n):
    x = wl.sweep_tokens(n, d, seed=100 + d + b, dtype=dtype)
    x[3] = 0  # a zero vector
    with kvq.Handle(d, b, 5, qjl=qjl) as h:
        codes, qj, norms = run_quantize(h, x.cuda())
    k = constants(d, b, 5)
    compare_quantize(k, x.double().numpy(), to_np_u32(codes), to_np_u32(qj) if qjl else None,
                     to_np_f16bits(norms), qjl)
    assert (to_np_u32(codes).reshape(n, -1)[3] == 0).all()
    assert (to_np_f16bits(norms).reshape(n, 2)[3] == 0).all()


BLOCK_CASES = [
    (128, 2, True, torch.bfloat16, 1000),
    (128, 1, False, torch.float16, 70),
    (64, 2, True, torch.float32, 333),
    (64, 4, True, torch.bfloat16, 31),
    (256, 2, True, torch.bfloat16, 300),
    (256, 3, False, torch.bfloat16, 129),
]


@pytest.mark.parametrize("d,b,qjl,dtype,n", BLOCK_CASES)
def test_quantize_block32_layout_matches_oracle(d, b, qjl, dtype, n):
    x = wl.sweep_tokens(n, d, seed=200 + d + b, dtype=dtype)
    x[min(5, n - 1)] = 0
    with kvq.Handle(d, b, 6, qjl=qjl) as h:
        codes, qj, norms = run_quantize(h, x.cuda(), layout=1)
        # the same bits as the token layout
        c0, q0, _ = run_quantize(h, x.cuda(), layout=0)
    k = constants(d, b, 6)
    compare_quantize(k, x.double().numpy(), to_np_u32(codes), to_np_u32(qj) if qjl else None,
                     to_np_f16bits(norms), qjl, layout=1)
    np.testing.assert_array_equal(oracle.unpack_codes_block32(to_np_u32(codes), b, d, n),
                                  oracle.unpack_codes(to_np_u32(c0).reshape(n, -1), b, d))
    if qjl:
        np.testing.assert_array_equal(oracle.unpack_bits_block32(to_np_u32(qj), d, n),
                                      oracle.unpack_bits(to_np_u32(q0).reshape(n, -1), d))
    # bits of vectors past n in the last block are zero
    tail = n % 32
    if tail:
        w = to_np_u32(codes)[-1]
        assert np.all((w >> np.uint32(tail)) == 0)


def test_strided_rows_and_single_vector():
    d = 128
    base = wl.llama_keys(1, 300, 192, seed=3)[0]  # rows of 192, use the first 128 columns
    x = base[:, :d]
    with kvq.Handle(d, 2, 9, qjl=True) as h:
        codes, qjl, norms = run_quantize(h, x.cuda())
        c1, q1, n1 = run_quantize(h, x[:1].contiguous().cuda())
    k = constants(d, 2, 9)
    compare_quantize(k, x.double().numpy(), to_np_u32(codes), to_np_u32(qjl), to_np_f16bits(norms), True)
    assert np.array_equal(to_np_u32(c1), to_np_u32(codes)[:1])
    assert np.array_equal(to_np_u32(q1), to_np_u32(qjl)[:1])


def test_empty_input_is_a_no_op():
    with kvq.Handle(128, 2, 1, qjl=True) as h:
        codes, qjl, norms = kvq.alloc_packed(h, 1)
        codes.fill_(7)
        kvq.kvq_quantize(h, torch.empty(0, 128, device="cuda", dtype=torch.bfloat16), codes, qjl, norms)
        assert kvq.kvq_status(h)[0] == 0
        assert (codes == 7).all()


def test_nonfinite_input_sets_status():
    with kvq.Handle(128, 2, 1, qjl=True) as h:
        x = torch.randn(256, 128, device="cuda")
        x[17, 5] = float("nan")
        codes, qjl, norms = kvq.alloc_packed(h, 256)
        kvq.kvq_quantize(h, x, codes, qjl, norms)
        code, bits = kvq.kvq_status(h)
        assert code == kvq.KVQ_ENONFINITE and bits & kvq.STATUS_NONFINITE
        # the status word is cleared by the read
        kvq.kvq_quantize(h, torch.randn(256, 128, device="cuda"), codes, qjl, norms)
        assert kvq.kvq_status(h)[0] == 0


def test_host_side_argument_errors():
    with kvq.Handle(128, 2, 1, qjl=True) as h:
        codes, qjl, norms = kvq.alloc_packed(h, 16)
        x = torch.randn(16, 128, device="cuda")
        # misaligned x, missing qjl on a QJL handle, row stride not a multiple of 16 bytes
        code = kvq.load().kvq_quantize(h.ptr, x.data_ptr() + 4, 0, 16, 128, 0, codes.data_ptr(), qjl.data_ptr(),
                                       norms.data_ptr(), None)
        assert code == kvq.KVQ_EINVAL
        code = kvq.load().kvq_quantize(h.ptr, x.data_ptr(), 0, 16, 128, 0, codes.data_ptr(), None,
                                       norms.data_ptr(), None)
        assert code == kvq.KVQ_EINVAL
        code = kvq.load().kvq_quantize(h.ptr, x.data_ptr(), 0, 16, 130, 0, codes.data_ptr(), qjl.data_ptr(),
                                       norms.data_ptr(), None)
        assert code == kvq.KVQ_EINVAL
        code = kvq.load().kvq_quantize(h.ptr, x.data_ptr(), 0, 16, 128, 2, codes.data_ptr(), qjl.data_ptr(),
                                       norms.data_ptr(), None)
        assert code == kvq.KVQ_EINVAL
        with pytest.raises(ValueError):
            kvq.kvq_quantize(h, x[:, :64], codes, qjl, norms)
    assert kvq.load().kvq_nsn_quantize(h.ptr if False else None, None, 0, 1, 128, 0, None, None, None, None) \
        == kvq.KVQ_EINVAL


def test_llama_layer_full_size_sampled():
    """8 KV heads x 32768 tokens x 128, bf16 keys with outlier channels, b=2 + QJL; oracle on sampled rows."""
    c = wl.LLAMA_LAYER
    K = wl.llama_keys(c["heads"], c["tokens"], c["d"], c["k_seed"], device="cuda")
    V = wl.llama_values(c["heads"], c["tokens"], c["d"], c["v_seed"], device="cuda")
    k = constants(c["d"], c["b"], c["handle_seed"])
    rng = np.random.default_rng(0)
    with kvq.Handle(c["d"], c["b"], c["handle_seed"], qjl=True) as h:
        # K and V of the layer in one fused launch, as the benchmark times them
        outs = [kvq.alloc_packed(h, K.numel() // c["d"], layout=lay) for lay in (0, 1)]
        kvq.kvq_quantize_batch(h, [(K, *outs[0], 0), (V, *outs[1], 1)])
        code, bits = kvq.kvq_status(h)
        assert code == 0, (code, bits)
        for X, layout in ((K, 0), (V, 1)):
            X2 = X.reshape(-1, c["d"])
            codes, qjl, norms = outs[layout]
            if layout == 0:
                idx = np.sort(rng.choice(X2.shape[0], 2048, replace=False))
                ti = torch.from_numpy(idx).cuda()
                compare_quantize(k, X2[ti].double().cpu().numpy(), to_np_u32(codes[ti]), to_np_u32(qjl[ti]),
                                 to_np_f16bits(norms[ti]), True)
            else:
                # sampled whole blocks of 32 vectors
                for blk in np.sort(rng.choice(X2.shape[0] // 32, 64, replace=False)):
                    sl = slice(blk * 32, blk * 32 + 32)
                    compare_quantize(k, X2[sl].double().cpu().numpy(), to_np_u32(codes[blk:blk + 1]),
                                     to_np_u32(qjl[blk:blk + 1]), to_np_f16bits(norms[sl]), True, layout=1)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("b", [1, 2, 3, 4])
@pytest.mark.parametrize("qjl", [True, False])
def test_sweep_full_size_sampled(d, b, qjl):
    """1,048,576 bf16 N(0,1) vectors with 1% of tokens x10; oracle on 256 sampled rows."""
    n = wl.SWEEP["n"]
    x = wl.sweep_tokens(n, d, seed=wl.SWEEP["seed"] + d, device="cuda")
    k = constants(d, b, wl.SWEEP["handle_seed"])
    with kvq.Handle(d, b, wl.SWEEP["handle_seed"], qjl=qjl) as h:
        codes, qj, norms = run_quantize(h, x)
    idx = np.sort(np.random.default_rng(d * 10 + b).choice(n, 256, replace=False))
    idx[-1] = n - 1
    ti = torch.from_numpy(idx).cuda()
    compare_quantize(k, x[ti].double().cpu().numpy(), to_np_u32(codes[ti]), to_np_u32(qj[ti]) if qjl else None,
                     to_np_f16bits(norms[ti]), qjl)


BATCH_CASES = [
    # d, b, qjl, (dtype, n, layout) of the first and of the second job
    (128, 2, True, (torch.bfloat16, 1000, 0), (torch.bfloat16, 300, 1)),  # one fused launch, ragged tails
    (64, 1, False, (torch.float16, 129, 1), (torch.float16, 2000, 0)),    # fused, block-32 first
    (128, 4, True, (torch.bfloat16, 31, 0), (torch.bfloat16, 33, 1)),     # fused, both under one tile
    (128, 3, True, (torch.bfloat16, 515, 0), (torch.float16, 257, 1)),    # dtypes differ: two launches
    (256, 2, True, (torch.bfloat16, 300, 0), (torch.bfloat16, 300, 1)),   # d = 256 with QJL: two launches
    (256, 4, False, (torch.float16, 700, 1), (torch.float16, 129, 0)),    # d = 256 without QJL: fused
    (128, 2, False, (torch.float32, 100, 0), (torch.float32, 70, 1)),     # fp32: two launches
]


@pytest.mark.parametrize("d,b,qjl,j0,j1", BATCH_CASES)
def test_quantize_batch_matches_oracle_and_single_calls(d, b, qjl, j0, j1):
    xs = [wl.sweep_tokens(n, d, seed=300 + d + b + i, dtype=dt) for i, (dt, n, _) in enumerate((j0, j1))]
    xs[0][min(2, j0[1] - 1)] = 0
    k = constants(d, b, 8)
    with kvq.Handle(d, b, 8, qjl=qjl) as h:
        outs = [kvq.alloc_packed(h, x.shape[0], layout=j[2]) for x, j in zip(xs, (j0, j1))]
        kvq.kvq_quantize_batch(h, [(x.cuda(), *o, j[2]) for x, o, j in zip(xs, outs, (j0, j1))])
        code, bits = kvq.kvq_status(h)
        assert code == 0, (code, bits)
        for x, (codes, qj, norms), j in zip(xs, outs, (j0, j1)):
            compare_quantize(k, x.double().numpy(), to_np_u32(codes), to_np_u32(qj) if qjl else None,
                             to_np_f16bits(norms), qjl, layout=j[2])
            # bit for bit what one kvq_quantize call per job writes
            c1, q1, n1 = run_quantize(h, x.cuda(), layout=j[2])
            assert torch.equal(c1, codes) and torch.equal(n1, norms)
            if qjl:
                assert torch.equal(q1, qj)


@pytest.mark.parametrize("d,b,qjl,dtype,n,layout", [
    (128, 2, True, torch.bfloat16, 1000, 0),
    (128, 2, True, torch.bfloat16, 777, 1),
    (64, 3, False, torch.float16, 257, 0),
    (128, 4, True, torch.float16, 300, 0),
    (64, 1, True, torch.bfloat16, 129, 1),
    (256, 2, False, torch.bfloat16, 300, 0),
    (256, 3, False, torch.float16, 129, 1),
])
def test_cuda_core_rotation_matches_oracle(d, b, qjl, dtype, n, layout):
    """KVQ_CUDA_CORE_ROTATION: 16-bit input, wherever the tensor-core rotation would run (d <= 128, and d = 256
    without QJL), through the in-register transform kernel, under the same parity rules; a layer's K and V
    through kvq_quantize_batch (one launch per job)."""
    x = wl.sweep_tokens(n, d, seed=500 + d + b, dtype=dtype)
    x[1] = 0
    k = constants(d, b, 9)
    with kvq.Handle(d, b, 9, qjl=qjl, cuda_core_rotation=True) as h:
        codes, qj, norms = run_quantize(h, x.cuda(), layout=layout)
        compare_quantize(k, x.double().numpy(), to_np_u32(codes), to_np_u32(qj) if qjl else None,
                         to_np_f16bits(norms), qjl, layout=layout)
        y = wl.sweep_tokens(n + 64, d, seed=600 + d + b, dtype=dtype)
        outs = [kvq.alloc_packed(h, t.shape[0], layout=lay) for t, lay in ((x, 0), (y, 1))]
        kvq.kvq_quantize_batch(h, [(t.cuda(), *o, lay) for t, o, lay in zip((x, y), outs, (0, 1))])
        code, bits = kvq.kvq_status(h)
        assert code == 0, (code, bits)
    for t, (c, q, nn), lay in zip((x, y), outs, (0, 1)):
        compare_quantize(k, t.double().numpy(), to_np_u32(c), to_np_u32(q) if qjl else None, to_np_f16bits(nn),
                         qjl, layout=lay)


def test_quantize_batch_empty_jobs_and_three_streams():
    d, b = 128, 2
    xs = [wl.sweep_tokens(n, d, seed=400 + n, dtype=torch.bfloat16) for n in (200, 0, 130, 64)]
    with kvq.Handle(d, b, 8, qjl=True) as h:
        lays = (0, 1, 1, 0)
        outs = [kvq.alloc_packed(h, max(x.shape[0], 1), layout=l) for x, l in zip(xs, lays)]
        kvq.kvq_quantize_batch(h, [(x.cuda(), *o, l) for x, o, l in zip(xs, outs, lays)])
        kvq.kvq_quantize_batch(h, [])
        assert kvq.kvq_status(h)[0] == 0
        for x, o, l in zip(xs, outs, lays):
            if x.shape[0] == 0:
                continue
            c1, q1, n1 = run_quantize(h, x.cuda(), layout=l)
            assert torch.equal(c1, o[0]) and torch.equal(q1, o[1]) and torch.equal(n1, o[2])


def test_quantize_batch_checks_every_job_before_launching():
    with kvq.Handle(128, 2, 1, qjl=True) as h:
        x = torch.randn(64, 128, device="cuda", dtype=torch.bfloat16)
        good = kvq.alloc_packed(h, 64)
        bad = kvq.alloc_packed(h, 64)
        good[0].fill_(7)
        jobs = (kvq.KvqQuantJob * 2)(kvq._job(h, x, *good, 0), kvq._job(h, x, *bad, 0))
        jobs[1].qjl = None  # a QJL handle needs the sign buffer
        code = kvq.load().kvq_quantize_batch(h.ptr, 2, jobs, None)
        assert code == kvq.KVQ_EINVAL
        assert kvq.load().kvq_last_error().decode().startswith("job 1")
        torch.cuda.synchronize()
        assert (good[0] == 7).all()  # nothing was launched
        assert kvq.load().kvq_quantize_batch(h.ptr, -1, None, None) == kvq.KVQ_EINVAL



@pytest.mark.parametrize("d,b,qjl,dtype,n", [
    (128, 2, True, torch.bfloat16, 1000),
    (64, 3, False, torch.float16, 300),
    (256, 4, True, torch.bfloat16, 257),
    (128, 1, False, torch.float32, 200),
    (128, 4, True, torch.bfloat16, 515),
])
def test_quantize_beta_codebook_matches_oracle(d, b, qjl, dtype, n):
    """KVQ_BETA_CODEBOOK: the kernels are unchanged, the codebook is the d-exact one."""
    x = wl.sweep_tokens(n, d, seed=500 + d + b, dtype=dtype)
    k = oracle.make_constants(d, b, 5, codebook="beta")
    with kvq.Handle(d, b, 5, qjl=qjl, beta=True) as h:
        _, _, cent, thr = kvq.kvq_get_constants(h)
        np.testing.assert_allclose(cent.numpy(), k.centroids, rtol=2.0 ** -23, atol=1e-12)
        np.testing.assert_allclose(thr.numpy(), k.thresholds, rtol=2.0 ** -23, atol=1e-12)
        codes, qj, norms = run_quantize(h, x.cuda())
    compare_quantize(k, x.double().numpy(), to_np_u32(codes), to_np_u32(qj) if qjl else None,
                     to_np_f16bits(norms), qjl)



def test_bounded_wait_runs_out_and_the_context_stays_usable():
    """A wait on an mbarrier nothing arrives on gives up after its poll bound: the status word
    reports the timeout (read on the host), and the next launches run normally."""
    with kvq.Handle(128, 2, 1, qjl=True) as h:
        kvq.kvq_probe_wait_timeout(h, 4096)
        code, bits = kvq.kvq_status(h)
        assert code == kvq.KVQ_ETIMEOUT and bits & kvq.STATUS_TIMEOUT
        x = wl.sweep_tokens(300, 128, seed=11)
        codes, qj, norms = run_quantize(h, x.cuda())
        compare_quantize(constants(128, 2, 1), x.double().numpy(), to_np_u32(codes), to_np_u32(qj),
                         to_np_f16bits(norms), True)
        with pytest.raises(kvq.KvqError):
            kvq.kvq_probe_wait_timeout(h, 0)


def test_size_limits_are_rejected_on_the_host():
    """More than 2^31 - 128 vectors in one call (the kernels index rows in 32 bits) is rejected
    before anything is read or launched, alone and inside a batch; so is a negative count."""
    with kvq.Handle(128, 2, 1, qjl=True) as h:
        L = kvq.load()
        big = (1 << 31) - 127
        assert L.kvq_quantize(h.ptr, None, kvq.KVQ_BF16, big, 128, 0, None, None, None, None) == kvq.KVQ_EINVAL
        assert "2^31" in kvq.kvq_last_error()
        assert L.kvq_quantize(h.ptr, None, kvq.KVQ_BF16, -1, 128, 0, None, None, None, None) == kvq.KVQ_EINVAL
        x = torch.randn(64, 128, device="cuda", dtype=torch.bfloat16)
        good = kvq.alloc_packed(h, 64)
        good[0].fill_(7)
        jobs = (kvq.KvqQuantJob * 2)(kvq._job(h, x, *good, 0), kvq._job(h, x, *good, 0))
        jobs[1].n = big
        assert L.kvq_quantize_batch(h.ptr, 2, jobs, None) == kvq.KVQ_EINVAL
        torch.cuda.synchronize()
        assert (good[0] == 7).all()
        # decode: hq not a multiple of hkv, and a GQA ratio that is not built
        out = torch.empty(1, 6, 128, device="cuda")
        ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
        c, qj, n = kvq.alloc_packed(h, 128)
        kc = kvq.make_cache(c, qj, n, 128, 0)
        vc_, vq_, vn_ = kvq.alloc_packed(h, 128, layout=1)
        vc = kvq.make_cache(vc_, vq_, vn_, 128, 1)
        sl = torch.tensor([128], dtype=torch.int32, device="cuda")
        q6 = torch.randn(1, 6, 128, device="cuda", dtype=torch.bfloat16)
        with pytest.raises(kvq.KvqError):
            kvq.kvq_decode_attend(h, q6, 4, kc, vc, sl, 128, 1.0, out, ws)
        q3 = torch.randn(1, 3, 128, device="cuda", dtype=torch.bfloat16)
        with pytest.raises(kvq.KvqError):  # hq / hkv = 3 is not built
            kvq.kvq_decode_attend(h, q3, 1, kc, vc, sl, 128, 1.0, out[:, :3], ws)
