"""Parity of the CUDA decode attention (through the C ABI) with the CPU oracle.

Both sides decode the same packed cache, the oracle's own quantization of
the seeded inputs, so only the attention arithmetic is compared."""
import numpy as np
import pytest
import torch

import oracle
from calibration_free_rotated_token_b200 import _abi as kvq
from calibration_free_rotated_token_b200 import workloads as wl

from .parity import assert_close, compare_quantize, oracle_cache, to_device_u32, to_np_f16bits, to_np_u32

pytestmark = pytest.mark.gpu

_consts = {}


def constants(d, b, seed, codebook="gaussian"):
    if (d, b, seed, codebook) not in _consts:
        _consts[(d, b, seed, codebook)] = oracle.make_constants(d, b, seed, codebook)
    return _consts[(d, b, seed, codebook)]


def upload_streams(h, caches, capacity, layout):
    """caches: list over streams of (codes, qjl, norms) numpy arrays -> device KvqCache + tensors."""
    S = len(caches)
    if layout == 0:
        codes = torch.zeros((S, capacity, h.b, h.d // 32), dtype=torch.int32, device="cuda")
        qjl = torch.zeros((S, capacity, h.m // 32), dtype=torch.int32, device="cuda") if h.qjl else None
    else:
        codes = torch.zeros((S, capacity // 32, h.b, h.d), dtype=torch.int32, device="cuda")
        qjl = torch.zeros((S, capacity // 32, h.m), dtype=torch.int32, device="cuda") if h.qjl else None
    norms = torch.zeros((S, capacity, 2), dtype=torch.float16, device="cuda")
    for s, (c, q, n) in enumerate(caches):
        T = n.shape[0]
        rows = c.shape[0]
        codes[s, :rows] = to_device_u32(c).reshape(codes[s, :rows].shape)
        if h.qjl:
            qjl[s, :rows] = to_device_u32(q).reshape(qjl[s, :rows].shape)
        norms[s, :T] = torch.from_numpy(np.ascontiguousarray(n)).cuda()
    return kvq.make_cache(codes, qjl, norms, capacity, layout), (codes, qjl, norms)


def run_decode(h, q, hkv, kc, vc, seq_len, max_T, scale, want_logits=True):
    B, hq, d = q.shape
    out = torch.empty((B, hq, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(kvq.kvq_decode_workspace(h, B, hq, hkv, max_T), dtype=torch.uint8, device="cuda")
    logits = torch.empty((B, hq, max_T), dtype=torch.float32, device="cuda") if want_logits else None
    sl = torch.tensor(seq_len, dtype=torch.int32, device="cuda")
    kvq.kvq_decode_attend(h, q, hkv, kc, vc, sl, max_T, scale, out, ws, logits)
    code, bits = kvq.kvq_status(h)
    assert code == 0, (code, bits)
    return out.cpu().numpy(), (logits.cpu().numpy() if want_logits else None)


def check_case(d, b, qjl, batch, hq, hkv, seq_len, capacity, scale, qdtype=torch.bfloat16, seed=3, beta=False):
    k = constants(d, b, seed, "beta" if beta else "gaussian")
    G = hq // hkv
    max_T = max(seq_len)
    kcs, vcs, kst, vst = [], [], [], []
    for bi in range(batch):
        for hk in range(hkv):
            T = seq_len[bi]
            K = wl.llama_keys(1, T, d, seed=1000 + bi * 31 + hk)[0].double().numpy()
            V = wl.llama_values(1, T, d, seed=2000 + bi * 31 + hk)[0].double().numpy()
            c, q, n, st = oracle_cache(k, K, qjl)
            kcs.append((c, q, n)); kst.append(st)
            c, q, n, st = oracle_cache(k, V, qjl, layout=1)
            vcs.append((c, q, n)); vst.append(st)
    qv = wl.queries(batch, hq, d, seed=77, dtype=qdtype)
    with kvq.Handle(d, b, seed, qjl=qjl, beta=beta) as h:
        kc, kt = upload_streams(h, kcs, capacity, 0)
        vc, vt = upload_streams(h, vcs, capacity, 1)
        out, logits = run_decode(h, qv.cuda(), hkv, kc, vc, seq_len, max_T, scale)
    qd = qv.double().numpy()
    for bi in range(batch):
        for hk in range(hkv):
            s = bi * hkv + hk
            lr, orf = oracle.decode_attend(k, qd[bi, hk * G:(hk + 1) * G], kst[s], vst[s], scale, qjl)
            assert_close(out[bi, hk * G:(hk + 1) * G], orf, f"out b{bi} kvh{hk}")
            T = seq_len[bi]
            if T > 0:
                assert_close(logits[bi, hk * G:(hk + 1) * G, :T], lr, f"logits b{bi} kvh{hk}")
            assert np.all(logits[bi, hk * G:(hk + 1) * G, T:] == -np.inf)


def test_tiny_reference_workload():
    """One query over 4096 fp32 N(0,1) keys/values, d=128, b=2 + QJL, scale 1/sqrt(128)."""
    c = wl.TINY
    k = constants(c["d"], c["b"], c["handle_seed"])
    K = wl.gaussian(c["n"], c["d"], c["data_seed"]).double().numpy()
    V = wl.gaussian(c["n"], c["d"], c["data_seed"] + 1000).double().numpy()
    ck, qk, nk, sk = oracle_cache(k, K, True)
    cv, qv_, nv, sv = oracle_cache(k, V, True, layout=1)
    q = wl.gaussian(1, c["d"], 7).reshape(1, 1, c["d"])
    with kvq.Handle(c["d"], c["b"], c["handle_seed"], qjl=True) as h:
        kc, _kt = upload_streams(h, [(ck, qk, nk)], c["n"], 0)
        vc, _vt = upload_streams(h, [(cv, qv_, nv)], c["n"], 1)
        out, logits = run_decode(h, q.cuda(), 1, kc, vc, [c["n"]], c["n"], c["scale"])
    lr, orf = oracle.decode_attend(k, q[0].double().numpy(), sk, sv, c["scale"], True)
    assert_close(logits[0], lr, "logits")
    assert_close(out[0], orf, "out")


@pytest.mark.parametrize("d,b,qjl,batch,hq,hkv,seq_len,cap,qdt", [
    (128, 2, True, 2, 8, 2, [1000, 777], 1120, torch.bfloat16),      # GQA 4:1, ragged contexts
    (128, 2, True, 1, 32, 8, [600], 608, torch.bfloat16),             # Llama-3-8B heads
    (128, 3, False, 2, 2, 2, [513, 1], 544, torch.float16),           # GQA 1:1, one-token context
    (64, 1, True, 1, 8, 1, [300], 320, torch.float32),                # GQA 8:1
    (64, 4, False, 2, 4, 2, [0, 257], 320, torch.bfloat16),           # an empty context
    (256, 2, True, 1, 4, 2, [400], 512, torch.bfloat16),
    (256, 4, False, 1, 2, 1, [129], 160, torch.bfloat16),
    (128, 1, False, 1, 2, 2, [300], 320, torch.bfloat16),            # tensor-core path, GQA 1:1
    (128, 2, False, 2, 4, 1, [900, 64], 960, torch.float16),          # tensor-core path without QJL
    (256, 1, True, 1, 4, 1, [700], 704, torch.bfloat16),              # d = 256, 1 bit: tensor-core path
    (256, 1, False, 2, 2, 2, [300, 45], 320, torch.float16),          # ... without QJL, ragged
    (256, 3, True, 1, 8, 2, [513], 544, torch.bfloat16),              # d = 256, 3 bits: CUDA-core path
    (256, 3, False, 2, 4, 4, [1, 260], 288, torch.bfloat16),          # ... one-token context
    (128, 4, True, 1, 8, 2, [600], 608, torch.bfloat16),              # 4 bits with QJL: CUDA-core path
    (64, 4, True, 2, 4, 1, [333, 0], 352, torch.float16),             # ... d = 64, an empty context
])
def test_decode_matches_oracle(d, b, qjl, batch, hq, hkv, seq_len, cap, qdt):
    check_case(d, b, qjl, batch, hq, hkv, seq_len, cap, scale=1 / np.sqrt(d), qdtype=qdt)


@pytest.mark.parametrize("d,b,qjl,batch,hq,hkv,seq_len,cap", [
    (128, 2, True, 2, 8, 2, [1000, 300], 1024),   # tensor-core path
    (64, 1, False, 1, 4, 4, [700], 704),          # tensor-core path, GQA 1:1
    (128, 3, True, 1, 4, 1, [513], 544),          # 3-bit path
    (256, 4, False, 1, 2, 1, [129], 160),
])
def test_decode_beta_codebook_matches_oracle(d, b, qjl, batch, hq, hkv, seq_len, cap):
    check_case(d, b, qjl, batch, hq, hkv, seq_len, cap, scale=1 / np.sqrt(d), beta=True)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("b", [1, 2, 3, 4])
@pytest.mark.parametrize("qjl", [True, False])
def test_decode_every_sweep_kernel(d, b, qjl):
    """Every (d, b, QJL) the sweep decodes, at its GQA 1:1 (one query per KV head): two sequences
    of 4500 and 4133 tokens (several splits and sub-chunks, ragged tails), logits and outputs."""
    check_case(d, b, qjl, 2, 1, 1, [4500, 4133], 4512, scale=1 / np.sqrt(d), qdtype=torch.bfloat16, seed=4)


def test_long_context_split_merge():
    """A context long enough for many splits (exact merge of the split partials)."""
    check_case(128, 2, True, 1, 4, 1, [20000], 20000, scale=1.0 / np.sqrt(128))


def _sampled_stream_decode(B, hq, hkv, T, sample, check_rows=1024, want_logits=True):
    """Cache of B x hkv streams of T tokens from the CUDA quantizer (Llama-layer generator);
    one sampled (sequence, KV head) is checked against the oracle's quantization on sampled
    rows and then replaced by the oracle's own cache, whose decode the oracle recomputes."""
    c = wl.DECODE
    d = c["d"]
    G = hq // hkv
    k = constants(d, c["b"], c["handle_seed"])
    with kvq.Handle(d, c["b"], c["handle_seed"], qjl=True) as h:
        S = B * hkv
        kcodes = torch.empty((S, T, h.b, d // 32), dtype=torch.int32, device="cuda")
        vcodes = torch.empty((S, T // 32, h.b, d), dtype=torch.int32, device="cuda")
        kqjl = torch.empty((S, T, d // 32), dtype=torch.int32, device="cuda")
        vqjl = torch.empty((S, T // 32, d), dtype=torch.int32, device="cuda")
        knorm = torch.empty((S, T, 2), dtype=torch.float16, device="cuda")
        vnorm = torch.empty_like(knorm)
        for bi in range(B):
            K = wl.llama_keys(hkv, T, d, wl.cache_slice_seed(c["handle_seed"], bi, 0, 0), device="cuda")
            V = wl.llama_values(hkv, T, d, wl.cache_slice_seed(c["handle_seed"], bi, 0, 1), device="cuda")
            sl = slice(bi * hkv, (bi + 1) * hkv)
            kvq.kvq_quantize(h, K, kcodes[sl], kqjl[sl], knorm[sl])
            for hk in range(hkv):
                kvq.kvq_quantize(h, V[hk], vcodes[bi * hkv + hk], vqjl[bi * hkv + hk], vnorm[bi * hkv + hk],
                                 layout=1)
            if bi == sample[0]:
                Ks = K[sample[1]].double().cpu().numpy()
                Vs = V[sample[1]].double().cpu().numpy()
        assert kvq.kvq_status(h)[0] == 0
        s = sample[0] * hkv + sample[1]
        rows = np.sort(np.random.default_rng(1).choice(T, min(check_rows, T), replace=False))
        tr = torch.from_numpy(rows).cuda()
        compare_quantize(k, Ks[rows], to_np_u32(kcodes[s][tr]), to_np_u32(kqjl[s][tr]),
                         to_np_f16bits(knorm[s][tr]), True)
        ck, qk, nk, sk = oracle_cache(k, Ks, True)
        cv, qv_, nv, sv = oracle_cache(k, Vs, True, layout=1)
        kcodes[s] = to_device_u32(ck).reshape(T, h.b, d // 32)
        kqjl[s] = to_device_u32(qk)
        knorm[s] = torch.from_numpy(nk).cuda()
        vcodes[s] = to_device_u32(cv).reshape(T // 32, h.b, d)
        vqjl[s] = to_device_u32(qv_)
        vnorm[s] = torch.from_numpy(nv).cuda()
        q = wl.queries(B, hq, d, c["q_seed"], device="cuda", std=c["q_std"])
        kc = kvq.make_cache(kcodes, kqjl, knorm, T, 0)
        vc = kvq.make_cache(vcodes, vqjl, vnorm, T, 1)
        out, logits = run_decode(h, q, hkv, kc, vc, [T] * B, T, c["scale"], want_logits=want_logits)
    qs = q[sample[0], sample[1] * G:(sample[1] + 1) * G].double().cpu().numpy()
    lr, orf = oracle.decode_attend(k, qs, sk, sv, c["scale"], True, want_logits=want_logits)
    assert_close(out[sample[0], sample[1] * G:(sample[1] + 1) * G], orf, "out (sampled stream)")
    if want_logits:
        assert_close(logits[sample[0], sample[1] * G:(sample[1] + 1) * G], lr, "logits (sampled stream)")
        assert np.isfinite(logits).all()
    assert np.isfinite(out).all()


def test_decode_several_subchunks_per_split():
    """4 sequences x 8 KV heads x 16384 tokens: 16 splits of 1024 tokens (four sub-chunks each)."""
    _sampled_stream_decode(4, 32, 8, 16384, sample=(2, 5))


def test_decode_workload_full_size_sampled():
    """batch 16, 32/8 heads, d 128, 131072-token contexts, b=2 + QJL, q ~ N(0,1)/sqrt(128), scale 1."""
    c = wl.DECODE
    _sampled_stream_decode(c["batch"], c["hq"], c["hkv"], c["T"], sample=(5, 3))


@pytest.mark.parametrize("d,b,qjl", [(64, 1, False), (64, 3, True), (128, 2, True), (128, 4, False),
                                     (256, 2, False), (256, 3, True), (256, 1, False)])
def test_sweep_decode_full_size_sampled(d, b, qjl):
    """Bit-width / head-dim sweep: the 1,048,576 bf16 vectors (1% x10) as 8 KV heads x 131072 tokens,
    quantized as K and V by the CUDA path, one N(0,1) query per KV head; one sampled head is checked
    against the oracle's quantization on sampled rows and then replaced by the oracle's own cache,
    whose decode the oracle recomputes."""
    c = wl.SWEEP
    H, T = c["hkv"], c["T"]
    k = constants(d, b, c["handle_seed"])
    X = wl.sweep_tokens(c["n"], d, seed=c["seed"] + d, device="cuda").reshape(H, T, d)
    Y = wl.sweep_tokens(c["n"], d, seed=c["seed"] + d + 500, device="cuda").reshape(H, T, d)
    hs = 3
    with kvq.Handle(d, b, c["handle_seed"], qjl=qjl) as h:
        kcodes, kqjl, knorm = kvq.alloc_packed(h, H * T)
        kvq.kvq_quantize(h, X.reshape(-1, d), kcodes, kqjl, knorm)
        vcodes = torch.empty((H, T // 32, b, d), dtype=torch.int32, device="cuda")
        vqjl = torch.empty((H, T // 32, d), dtype=torch.int32, device="cuda") if qjl else None
        vnorm = torch.empty((H, T, 2), dtype=torch.float16, device="cuda")
        for hk in range(H):
            kvq.kvq_quantize(h, Y[hk], vcodes[hk], vqjl[hk] if qjl else None, vnorm[hk], layout=1)
        assert kvq.kvq_status(h)[0] == 0
        kcodes = kcodes.reshape(H, T, b, d // 32)
        kqjl = kqjl.reshape(H, T, d // 32) if qjl else None
        knorm = knorm.reshape(H, T, 2)
        Xs = X[hs].double().cpu().numpy()
        Ys = Y[hs].double().cpu().numpy()
        rows = np.sort(np.random.default_rng(d + b).choice(T, 512, replace=False))
        tr = torch.from_numpy(rows).cuda()
        compare_quantize(k, Xs[rows], to_np_u32(kcodes[hs][tr]), to_np_u32(kqjl[hs][tr]) if qjl else None,
                         to_np_f16bits(knorm[hs][tr]), qjl)
        ck, qk, nk, sk = oracle_cache(k, Xs, qjl)
        cv, qv_, nv, sv = oracle_cache(k, Ys, qjl, layout=1)
        kcodes[hs] = to_device_u32(ck).reshape(T, b, d // 32)
        knorm[hs] = torch.from_numpy(nk).cuda()
        vcodes[hs] = to_device_u32(cv).reshape(T // 32, b, d)
        vnorm[hs] = torch.from_numpy(nv).cuda()
        if qjl:
            kqjl[hs] = to_device_u32(qk)
            vqjl[hs] = to_device_u32(qv_)
        q = wl.queries(1, H, d, seed=c["seed"] + 7, device="cuda")
        kc = kvq.make_cache(kcodes, kqjl, knorm, T, 0)
        vc = kvq.make_cache(vcodes, vqjl, vnorm, T, 1)
        out, _ = run_decode(h, q, H, kc, vc, [T], T, 1.0 / np.sqrt(d), want_logits=False)
    _, orf = oracle.decode_attend(k, q[0, hs:hs + 1].double().cpu().numpy(), sk, sv, 1.0 / np.sqrt(d), qjl,
                                  want_logits=False)
    assert_close(out[0, hs:hs + 1], orf, "out (sampled head)")
    assert np.isfinite(out).all()


def test_decode_more_than_512_splits():
    """One stream of 528384 tokens: the tensor-core path splits it into 516 items of 1024 tokens,
    so the combine merges more split partials than it caches at once.  The cache is the oracle's
    own quantization of 4096 seeded keys and values, repeated 129 times along the context."""
    d, b, rep = 128, 2, 129
    k = constants(d, b, 1)
    K = wl.sweep_tokens(4096, d, seed=601).double().numpy()
    V = wl.sweep_tokens(4096, d, seed=602).double().numpy()
    ck, qk, nk, sk = oracle_cache(k, K, True)
    cv, qv, nv, sv = oracle_cache(k, V, True, layout=1)
    T = 4096 * rep
    tile = lambda a: np.concatenate([a] * rep, axis=0)
    kst = {key: tile(v) for key, v in sk.items()}
    vst = {key: tile(v) for key, v in sv.items()}
    q = wl.queries(1, 1, d, seed=603)
    with kvq.Handle(d, b, 1, qjl=True) as h:
        kc, _kt = upload_streams(h, [(tile(ck), tile(qk), tile(nk))], T, 0)
        vc, _vt = upload_streams(h, [(tile(cv), tile(qv), tile(nv))], T, 1)
        out, _ = run_decode(h, q.cuda(), 1, kc, vc, [T], T, 1 / np.sqrt(d), want_logits=False)
    _, orf = oracle.decode_attend(k, q[0].double().numpy(), kst, vst, 1 / np.sqrt(d), True, want_logits=False)
    assert_close(out[0], orf, "out over 516 splits")
