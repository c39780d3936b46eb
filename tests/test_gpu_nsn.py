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

from .parity import CODE_BAND, assert_close, pool_add, to_np_f16bits, to_np_u32, ulp_distance_f16

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


def check_head(k, x, codes_g, norms_g, means_g, pool=None):
    """x: [T, d] float64 of one head; GPU outputs of that head.  The boundary-excluded count
    goes to the workload `pool` (see parity.pooled_check)."""
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
    if pool is not None:
        pool_add(pool, near.sum(), near.size)
    nb = norms_g.reshape(T, 2)
    assert ulp_distance_f16(nb[:, 0], ref["norm_x"].astype(np.float16).view(np.uint16)).max() <= 1
    ok = ~near.any(1)
    assert ulp_distance_f16(nb[ok, 1], ref["norm_w"][ok].astype(np.float16).view(np.uint16)).max(initial=0) <= 1
    stats["excluded_coords"] = int(near.sum())
    return stats


@pytest.mark.parametrize("d,b,dtype", [(128, 2, torch.bfloat16), (128, 1, torch.float16), (64, 3, torch.float32),
                                       (64, 4, torch.bfloat16),
                                       # d = 256: the rotation as two 128-wide tensor-core products
                                       (256, 2, torch.bfloat16), (256, 3, torch.float16), (256, 4, torch.bfloat16)])
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


@pytest.mark.parametrize("d", [128, 256])
def test_nsn_block32_layout_matches_token_layout(d):
    """Values are stored in the block-32 layout: the same bits, norms and block means."""
    b = 2
    x = wl.nsn_tokens(2, 256, d, seed=9).cuda()
    with kvq.Handle(d, b, 3, qjl=False) as h:
        c0, n0, m0 = run_nsn(h, x)
        c1 = torch.empty((2, 256 // 32, b, d), dtype=torch.int32, device="cuda")
        n1 = torch.empty_like(n0)
        m1 = torch.empty_like(m0)
        kvq.kvq_nsn_quantize(h, x, c1, n1, m1, layout=kvq.KVQ_LAYOUT_BLOCK32)
        assert kvq.kvq_status(h)[0] == 0
    for hh in range(2):
        np.testing.assert_array_equal(oracle.unpack_codes_block32(to_np_u32(c1[hh]), b, d, 256),
                                      oracle.unpack_codes(to_np_u32(c0[hh]).reshape(256, -1), b, d))
    assert torch.equal(n0, n1) and torch.equal(m0, m1)


# ---------------------------------------------------------------------------
# Decode attention over NSN caches (kvq_nsn_decode_attend)
# ---------------------------------------------------------------------------
def _nsn_oracle_stream(k, X):
    """The oracle's NSN cache of one stream X [T, d] (T % 128 == 0): packed key and value
    records, norms, block means, and the stored values the oracle decodes from."""
    r = oracle.nsn_quantize(k, X)
    nb = np.stack([r["norm_x"].astype(np.float16), r["norm_w"].astype(np.float16)], axis=1)
    stored = dict(codes=r["codes"], norm_x=nb[:, 0].astype(np.float64), norm_w=nb[:, 1].astype(np.float64))
    return r, nb, stored


def check_nsn_decode(d, b, batch, hq, hkv, seq_len, cap, qdtype=torch.bfloat16, seed=5):
    k = oracle.make_constants(d, b, seed)
    G = hq // hkv
    S = batch * hkv
    kc = torch.zeros((S, cap, b, d // 32), dtype=torch.int32)
    vc = torch.zeros((S, cap // 32, b, d), dtype=torch.int32)
    kn = torch.zeros((S, cap, 2), dtype=torch.float16)
    vn = torch.zeros_like(kn)
    km = torch.zeros((S, cap // 128, d), dtype=torch.float16)
    vm = torch.zeros_like(km)
    kst, vst = [], []
    for s in range(S):
        K = wl.nsn_tokens(1, cap, d, seed=700 + s)[0].double().numpy()
        V = wl.nsn_tokens(1, cap, d, seed=900 + s)[0].double().numpy()
        rk, nbk, sk = _nsn_oracle_stream(k, K)
        rv, nbv, sv = _nsn_oracle_stream(k, V)
        kc[s] = torch.from_numpy(oracle.pack_codes(rk["codes"], b).view(np.int32))
        vc[s] = torch.from_numpy(oracle.pack_codes_block32(rv["codes"], b).view(np.int32).reshape(cap // 32, b, d))
        kn[s] = torch.from_numpy(nbk)
        vn[s] = torch.from_numpy(nbv)
        km[s] = torch.from_numpy(rk["mean_half"].view(np.float16))
        vm[s] = torch.from_numpy(rv["mean_half"].view(np.float16))
        kst.append((sk, rk["mean_half"]))
        vst.append((sv, rv["mean_half"]))
    q = wl.queries(batch, hq, d, seed=77, dtype=qdtype)
    scale = 1 / np.sqrt(d)
    max_T = max(seq_len)
    with kvq.Handle(d, b, seed, qjl=False) as h:
        kcd, vcd, knd, vnd, kmd, vmd = (t.cuda() for t in (kc, vc, kn, vn, km, vm))
        kcache = kvq.make_cache(kcd, None, knd, cap, 0)
        vcache = kvq.make_cache(vcd, None, vnd, cap, 1)
        out = torch.empty((batch, hq, d), dtype=torch.float32, device="cuda")
        logits = torch.empty((batch, hq, max_T), dtype=torch.float32, device="cuda")
        ws = torch.empty(kvq.kvq_decode_workspace(h, batch, hq, hkv, max_T), dtype=torch.uint8, device="cuda")
        sl = torch.tensor(seq_len, dtype=torch.int32, device="cuda")
        kvq.kvq_nsn_decode_attend(h, q.cuda(), hkv, kcache, vcache, kmd, vmd, sl, max_T, scale, out, ws, logits)
        code, bits = kvq.kvq_status(h)
        assert code == 0, (code, bits)
        out, logits = out.cpu().numpy(), logits.cpu().numpy()
    qd = q.double().numpy()
    for bi in range(batch):
        T = seq_len[bi]
        nblk = (T + 127) // 128
        for hk in range(hkv):
            s = bi * hkv + hk
            sk = {key: v[:T] for key, v in kst[s][0].items()}
            sv = {key: v[:T] for key, v in vst[s][0].items()}
            lr, orf = oracle.nsn_decode_attend(k, qd[bi, hk * G:(hk + 1) * G], sk, sv, kst[s][1][:nblk],
                                               vst[s][1][:nblk], scale)
            assert_close(out[bi, hk * G:(hk + 1) * G], orf, f"nsn out b{bi} kvh{hk}")
            if T > 0:
                assert_close(logits[bi, hk * G:(hk + 1) * G, :T], lr, f"nsn logits b{bi} kvh{hk}")
            assert np.all(logits[bi, hk * G:(hk + 1) * G, T:] == -np.inf)


@pytest.mark.parametrize("d,b,batch,hq,hkv,seq_len,cap", [
    (128, 2, 2, 8, 2, [1000, 300], 1024),    # GQA 4:1, ragged contexts, partial blocks
    (64, 1, 1, 4, 4, [640], 640),            # GQA 1:1
    (128, 2, 1, 16, 2, [2000], 2048),        # GQA 8:1
    (256, 2, 1, 4, 2, [513], 640),           # 128-token sub-chunks (one block each)
    (128, 1, 2, 4, 1, [0, 129], 256),        # an empty context
    (128, 3, 1, 8, 2, [700], 768),           # 3 bits (parity plane)
    (64, 3, 1, 4, 1, [384], 384),
    # CUDA-core path (4-bit codebooks, 3 bits at d = 256)
    (128, 4, 2, 8, 2, [1000, 300], 1024),    # GQA 4:1, ragged contexts, partial blocks
    (64, 4, 1, 4, 4, [640], 640),            # GQA 1:1
    (256, 3, 1, 8, 1, [700], 768),           # GQA 8:1, 128-token tiles
    (256, 4, 2, 4, 2, [0, 300], 384),        # an empty context
])
def test_nsn_decode_matches_oracle(d, b, batch, hq, hkv, seq_len, cap):
    check_nsn_decode(d, b, batch, hq, hkv, seq_len, cap)


def test_nsn_decode_long_context():
    """Many splits merged exactly, the block-mean term included."""
    check_nsn_decode(128, 2, 1, 4, 1, [20480], 20480)


def test_nsn_decode_workload_full_size_sampled():
    """The NSN workload (8 heads x 65536 tokens, b=2) quantized by the CUDA NSN front end, keys per
    token and values in blocks of 32, then decoded by 32 query heads (GQA 4:1, one token).  One
    sampled KV head is checked against the oracle's NSN quantization on sampled blocks and then
    replaced by the oracle's own NSN cache, whose decode the oracle recomputes."""
    c = wl.NSN
    H, T, d, b = c["heads"], c["tokens"], c["d"], c["b"]
    hs = 5
    k = oracle.make_constants(d, b, c["handle_seed"])
    X = wl.nsn_tokens(H, T, d, c["seed"], device="cuda")
    Y = wl.nsn_tokens(H, T, d, c["seed"] + 1, device="cuda")
    with kvq.Handle(d, b, c["handle_seed"], qjl=False) as h:
        kc = torch.empty((H, T, h.b, d // 32), dtype=torch.int32, device="cuda")
        vc = torch.empty((H, T // 32, h.b, d), dtype=torch.int32, device="cuda")
        kn = torch.empty((H, T, 2), dtype=torch.float16, device="cuda")
        vn = torch.empty_like(kn)
        km = torch.empty((H, T // 128, d), dtype=torch.float16, device="cuda")
        vm = torch.empty_like(km)
        kvq.kvq_nsn_quantize(h, X, kc, kn, km)
        kvq.kvq_nsn_quantize(h, Y, vc, vn, vm, layout=kvq.KVQ_LAYOUT_BLOCK32)
        assert kvq.kvq_status(h)[0] == 0
        Xs = X[hs].double().cpu().numpy()
        Ys = Y[hs].double().cpu().numpy()
        for blk in (0, 77, T // 128 - 1):  # the CUDA records of the sampled head, against the oracle
            sl = slice(blk * 128, (blk + 1) * 128)
            check_head(k, Xs[sl], to_np_u32(kc[hs, sl]), to_np_f16bits(kn[hs, sl]), to_np_f16bits(km[hs, blk:blk + 1]))
        # the sampled head's cache becomes the oracle's own
        rk, nbk, sk = _nsn_oracle_stream(k, Xs)
        rv, nbv, sv = _nsn_oracle_stream(k, Ys)
        kc[hs] = torch.from_numpy(oracle.pack_codes(rk["codes"], b).view(np.int32)).cuda()
        vc[hs] = torch.from_numpy(oracle.pack_codes_block32(rv["codes"], b).view(np.int32).reshape(T // 32, b, d)).cuda()
        kn[hs] = torch.from_numpy(nbk).cuda()
        vn[hs] = torch.from_numpy(nbv).cuda()
        km[hs] = torch.from_numpy(rk["mean_half"].view(np.float16)).cuda()
        vm[hs] = torch.from_numpy(rv["mean_half"].view(np.float16)).cuda()
        q = wl.queries(1, 4 * H, d, seed=78, device="cuda")
        out = torch.empty((1, 4 * H, d), dtype=torch.float32, device="cuda")
        ws = torch.empty(kvq.kvq_decode_workspace(h, 1, 4 * H, H, T), dtype=torch.uint8, device="cuda")
        sl = torch.tensor([T], dtype=torch.int32, device="cuda")
        kvq.kvq_nsn_decode_attend(h, q, H, kvq.make_cache(kc, None, kn, T, 0), kvq.make_cache(vc, None, vn, T, 1),
                                  km, vm, sl, T, d ** -0.5, out, ws)
        assert kvq.kvq_status(h)[0] == 0
    qd = q.double().cpu().numpy()
    out = out.cpu().numpy()
    _, orf = oracle.nsn_decode_attend(k, qd[0, 4 * hs:4 * hs + 4], sk, sv, rk["mean_half"], rv["mean_half"],
                                      d ** -0.5, want_logits=False)
    assert_close(out[0, 4 * hs:4 * hs + 4], orf, f"nsn workload out kvh{hs}")
    assert np.isfinite(out).all()


def test_nsn_front_end_at_d256_rejects_fp32():
    with kvq.Handle(256, 2, 3, qjl=False) as h:
        x = torch.randn(1, 128, 256, device="cuda", dtype=torch.float32)
        with pytest.raises(kvq.KvqError) as e:
            run_nsn(h, x)
        assert e.value.code == kvq.KVQ_EUNSUPPORTED
