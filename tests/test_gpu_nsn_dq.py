"""Parity of the double-quantized NSN front end and of decode over its caches
(through the C ABI) with the CPU oracle (NSNQuant summary, section 3,
"Double Quantization"; the record format is stated in include/kvq.h).

The GPU takes each rounding decision of the side record (the fp16 steps and
offset, the 4-bit codes) in fp32, the oracle in fp64.  A GPU decision that
differs must be the other neighbour at a near-tie of the oracle's value; the
oracle is then re-run with the GPU's record parts (oracle-derived values from
the same inputs), first the norm part -- from which the oracle recomputes the
means -- then the whole record, and the codes and ||w|| are compared with
the usual rules."""
import numpy as np
import pytest
import torch

import oracle
from calibration_free_rotated_token_b200 import _abi as kvq
from calibration_free_rotated_token_b200 import workloads as wl

from .parity import CODE_BAND, assert_close, pool_add, pooled_check, to_np_f16bits, to_np_u32, ulp_distance_f16

pytestmark = pytest.mark.gpu

TIE = 1e-5  # relative distance of a value from a rounding midpoint that counts as a near-tie


def _f16(rec, o):
    return rec[:, o:o + 2].copy().view(np.float16)[:, 0].astype(np.float64)


def _nib(rec, start, n):
    b = rec[:, start:start + n // 2]
    return np.stack([b & 15, b >> 4], axis=2).reshape(rec.shape[0], n).astype(np.int64)


def _f16_ok(got, exact):
    """got (fp16 value) is fp16(exact), or its other neighbour when exact is near a midpoint."""
    want = np.float16(exact).astype(np.float64)
    if got == want:
        return True
    lo, hi = sorted((got, want))
    mid = 0.5 * (lo + hi)
    return abs(np.nextafter(np.float16(lo), np.float16(np.inf)).astype(np.float64) - hi) == 0 and \
        abs(exact - mid) <= TIE * max(abs(exact), 1e-30)


def _codes_ok(got, v, lo_clamp, hi_clamp):
    """got: integer codes; v: the exact quotients they round (rint, then clamp)."""
    want = np.clip(np.rint(v), lo_clamp, hi_clamp)
    diff = got != want
    frac = np.abs(v - np.floor(v) - 0.5)
    tie = frac <= TIE * np.maximum(np.abs(v), 1.0)
    near = diff & tie & (np.abs(got - v) <= 0.5 + TIE * np.maximum(np.abs(v), 1.0))
    return np.all(~diff | near), int(diff.sum())


def check_dq_head(k, x, codes_g, wnorm_g, side_g, pool=None):
    """x: [T, d] float64 of one head (T % 128 == 0); the GPU's codes (token layout), fp16 ||w||
    bits and side records of that head."""
    T, d = x.shape
    side_g = np.asarray(side_g, np.uint8).reshape(T // 128, -1)
    own = oracle.nsn_dq_quantize(k, x)
    # norm part: step, then the codes on the GPU's step
    ns_g = _f16(side_g, 4)
    for bi in range(T // 128):
        assert _f16_ok(ns_g[bi], own["norm_x"][bi * 128:(bi + 1) * 128].max() / 15.0), f"norm step of block {bi}"
    qn_g = _nib(side_g, 8 + d // 2, 128)
    nx = own["norm_x"].reshape(-1, 128)
    v = np.where(ns_g[:, None] > 0, nx / np.where(ns_g[:, None] > 0, ns_g[:, None], 1.0), 0.0)
    nz = (nx > 0) & (ns_g[:, None] > 0)
    ok, nd_n = _codes_ok(qn_g[nz], v[nz], 1, 15)
    assert ok and np.all(qn_g[~nz] == 0), "norm codes differ away from a rounding tie"
    # mean part, with the oracle's means recomputed on the GPU's norm part
    ra = oracle.nsn_dq_quantize(k, x, side_in=side_g, parts=1)
    lo_g, st_g = _f16(side_g, 0), _f16(side_g, 2)
    of = ra["mean_f64"]
    for bi in range(T // 128):
        assert _f16_ok(lo_g[bi], of[bi].min()), f"mean offset of block {bi}"
        assert _f16_ok(st_g[bi], (of[bi].max() - of[bi].min()) / 15.0), f"mean step of block {bi}"
    qo_g = _nib(side_g, 8, d)
    vo = np.where(st_g[:, None] > 0, (of - lo_g[:, None]) / np.where(st_g[:, None] > 0, st_g[:, None], 1.0), 0.0)
    ok, nd_o = _codes_ok(qo_g, vo, 0, 15)
    assert ok, "mean codes differ away from a rounding tie"
    assert np.all(side_g[:, 6:8] == 0) and np.all(side_g[:, 8 + d // 2 + 64:] == 0), "record padding is not zero"
    # codes and ||w|| for the GPU's whole record
    ref = oracle.nsn_dq_quantize(k, x, side_in=side_g, parts=3)
    codes = oracle.unpack_codes(np.asarray(codes_g).reshape(T, -1), k.b, d)
    near = (np.abs(ref["z"][..., None] - k.thresholds) < CODE_BAND).any(-1)
    bad = (codes != ref["codes"]) & ~near
    assert bad.sum() == 0, f"{bad.sum()} codes differ outside the boundary band"
    if near.any():
        kk = np.argmin(np.abs(ref["z"][near][:, None] - k.thresholds[None, :]), axis=1)
        assert np.all((codes[near] == kk) | (codes[near] == kk + 1))
    if pool is not None:
        pool_add(pool, near.sum(), near.size)
    okv = ~near.any(1)
    dw = ulp_distance_f16(np.asarray(wnorm_g).reshape(T), ref["norm_w"].astype(np.float16).view(np.uint16))
    assert dw[okv].max(initial=0) <= 1, f"||w|| off by {dw[okv].max()} ulp"
    return dict(norm_code_ties=nd_n, mean_code_ties=nd_o, excluded=int(near.sum()))


def run_dq(h, x, layout=0):
    H, T, d = x.shape
    R = kvq.kvq_nsn_dq_side_bytes(d)
    if layout == 0:
        codes = torch.empty((H, T, h.b, d // 32), dtype=torch.int32, device="cuda")
    else:
        codes = torch.empty((H, T // 32, h.b, d), dtype=torch.int32, device="cuda")
    wn = torch.empty((H, T), dtype=torch.float16, device="cuda")
    side = torch.full((H, T // 128, R), 0xAB, dtype=torch.uint8, device="cuda")
    kvq.kvq_nsn_dq_quantize(h, x, codes, wn, side, layout=layout)
    code, bits = kvq.kvq_status(h)
    assert code == 0, (code, bits)
    return codes, wn, side


@pytest.mark.parametrize("d,b,dtype", [(128, 2, torch.bfloat16), (128, 1, torch.float16), (64, 3, torch.bfloat16),
                                       (64, 2, torch.float16), (128, 4, torch.bfloat16),
                                       # d = 256: the rotation as two 128-wide tensor-core products
                                       (256, 2, torch.bfloat16), (256, 4, torch.float16), (256, 1, torch.bfloat16)])
def test_nsn_dq_matches_oracle(d, b, dtype):
    x = wl.nsn_tokens(2, 512, d, seed=30 + d + b, dtype=dtype)
    x[1, 130] = 0  # a zero token inside a block
    x[0, 5] *= 1e-3  # a tiny token: the smallest nonzero norm code
    with kvq.Handle(d, b, 3, qjl=False) as h:
        codes, wn, side = run_dq(h, x.cuda())
    k = oracle.make_constants(d, b, 3)
    for hh in range(2):
        check_dq_head(k, x[hh].double().numpy(), to_np_u32(codes[hh]), to_np_f16bits(wn[hh]),
                      side[hh].cpu().numpy(), pool="nsn_dq")
    assert (_nib(side[1].cpu().numpy(), 8 + d // 2, 128)[1, 2] == 0)  # token 130 = block 1, row 2


@pytest.mark.parametrize("d", [128, 256])
def test_nsn_dq_block32_layout_matches_token_layout(d):
    b = 2
    x = wl.nsn_tokens(2, 256, d, seed=9).cuda()
    with kvq.Handle(d, b, 3, qjl=False) as h:
        c0, w0, s0 = run_dq(h, x)
        c1, w1, s1 = run_dq(h, x, layout=kvq.KVQ_LAYOUT_BLOCK32)
    for hh in range(2):
        np.testing.assert_array_equal(oracle.unpack_codes_block32(to_np_u32(c1[hh]), b, d, 256),
                                      oracle.unpack_codes(to_np_u32(c0[hh]).reshape(256, -1), b, d))
    assert torch.equal(w0, w1) and torch.equal(s0, s1)


def test_nsn_dq_rejects_unbuilt_and_invalid_calls():
    with kvq.Handle(128, 2, 3, qjl=False) as h:
        x = torch.randn(1, 128, 128, device="cuda", dtype=torch.float32)
        codes = torch.empty(128 * 8, dtype=torch.int32, device="cuda")
        wn = torch.empty(128, dtype=torch.float16, device="cuda")
        side = torch.empty(kvq.kvq_nsn_dq_side_bytes(128), dtype=torch.uint8, device="cuda")
        with pytest.raises(kvq.KvqError) as e:  # fp32 input is not built
            kvq.kvq_nsn_dq_quantize(h, x, codes, wn, side)
        assert e.value.code == kvq.KVQ_EUNSUPPORTED
        with pytest.raises(kvq.KvqError):  # ragged token count
            kvq.kvq_nsn_dq_quantize(h, torch.randn(1, 100, 128, device="cuda", dtype=torch.bfloat16), codes, wn,
                                    side)
    assert kvq.kvq_nsn_dq_side_bytes(128) == 144 and kvq.kvq_nsn_dq_side_bytes(64) == 112
    assert kvq.kvq_nsn_dq_side_bytes(256) == 208 and kvq.kvq_nsn_dq_side_bytes(96) == 0


def _dq_oracle_stream(k, X):
    r = oracle.nsn_dq_quantize(k, X)
    wnb = r["norm_w"].astype(np.float16)
    return r, wnb, dict(codes=r["codes"], norm_w=wnb.astype(np.float64))


def check_dq_decode(d, b, batch, hq, hkv, seq_len, cap, qdtype=torch.bfloat16, seed=5):
    k = oracle.make_constants(d, b, seed)
    G = hq // hkv
    S = batch * hkv
    R = oracle.nsn_dq_rec_bytes(d)
    kc = torch.zeros((S, cap, b, d // 32), dtype=torch.int32)
    vc = torch.zeros((S, cap // 32, b, d), dtype=torch.int32)
    kn = torch.zeros((S, cap), dtype=torch.float16)
    vn = torch.zeros_like(kn)
    ks = torch.zeros((S, cap // 128, R), dtype=torch.uint8)
    vs = torch.zeros_like(ks)
    kst, vst = [], []
    for s in range(S):
        rk, wk, sk = _dq_oracle_stream(k, wl.nsn_tokens(1, cap, d, seed=700 + s)[0].double().numpy())
        rv, wv, sv = _dq_oracle_stream(k, wl.nsn_tokens(1, cap, d, seed=900 + s)[0].double().numpy())
        kc[s] = torch.from_numpy(oracle.pack_codes(rk["codes"], b).view(np.int32))
        vc[s] = torch.from_numpy(oracle.pack_codes_block32(rv["codes"], b).view(np.int32).reshape(cap // 32, b, d))
        kn[s] = torch.from_numpy(wk)
        vn[s] = torch.from_numpy(wv)
        ks[s] = torch.from_numpy(rk["side"])
        vs[s] = torch.from_numpy(rv["side"])
        kst.append((sk, rk["side"]))
        vst.append((sv, rv["side"]))
    q = wl.queries(batch, hq, d, seed=77, dtype=qdtype)
    scale = 1 / np.sqrt(d)
    max_T = max(seq_len)
    with kvq.Handle(d, b, seed, qjl=False) as h:
        kcd, vcd, knd, vnd, ksd, vsd = (t.cuda() for t in (kc, vc, kn, vn, ks, vs))
        kcache = kvq.make_cache(kcd, None, knd, cap, 0)
        vcache = kvq.make_cache(vcd, None, vnd, cap, 1)
        out = torch.empty((batch, hq, d), dtype=torch.float32, device="cuda")
        logits = torch.empty((batch, hq, max_T), dtype=torch.float32, device="cuda")
        ws = torch.empty(kvq.kvq_decode_workspace(h, batch, hq, hkv, max_T), dtype=torch.uint8, device="cuda")
        sl = torch.tensor(seq_len, dtype=torch.int32, device="cuda")
        kvq.kvq_nsn_dq_decode_attend(h, q.cuda(), hkv, kcache, vcache, ksd, vsd, sl, max_T, scale, out, ws, logits)
        code, bits = kvq.kvq_status(h)
        assert code == 0, (code, bits)
        out, logits = out.cpu().numpy(), logits.cpu().numpy()
    qd = q.double().numpy()
    for bi in range(batch):
        T = seq_len[bi]
        for hk in range(hkv):
            s = bi * hkv + hk
            sk = {key: v[:T] for key, v in kst[s][0].items()}
            sv = {key: v[:T] for key, v in vst[s][0].items()}
            lr, orf = oracle.nsn_dq_decode_attend(k, qd[bi, hk * G:(hk + 1) * G], sk, sv, kst[s][1], vst[s][1], scale)
            assert_close(out[bi, hk * G:(hk + 1) * G], orf, f"nsn-dq out b{bi} kvh{hk}")
            if T > 0:
                assert_close(logits[bi, hk * G:(hk + 1) * G, :T], lr, f"nsn-dq logits b{bi} kvh{hk}")
            assert np.all(logits[bi, hk * G:(hk + 1) * G, T:] == -np.inf)


@pytest.mark.parametrize("d,b,batch,hq,hkv,seq_len,cap", [
    (128, 2, 2, 8, 2, [1000, 300], 1024),    # GQA 4:1, ragged contexts, partial blocks
    (64, 1, 1, 4, 4, [640], 640),            # GQA 1:1
    (128, 2, 1, 16, 2, [2000], 2048),        # GQA 8:1
    (128, 1, 2, 4, 1, [0, 129], 256),        # an empty context
    (128, 3, 1, 8, 2, [700], 768),           # 3 bits (parity plane)
    (256, 2, 1, 4, 2, [513], 640),           # d = 256 on the tensor cores (128-token sub-chunks)
    # CUDA-core path: 4-bit codebooks, 3 bits at d = 256
    (128, 4, 2, 8, 2, [1000, 300], 1024),
    (64, 4, 1, 4, 4, [640], 640),
    (256, 3, 2, 4, 1, [0, 700], 768),        # an empty context
])
def test_nsn_dq_decode_matches_oracle(d, b, batch, hq, hkv, seq_len, cap):
    check_dq_decode(d, b, batch, hq, hkv, seq_len, cap)


def test_nsn_dq_decode_long_context():
    check_dq_decode(128, 2, 1, 4, 1, [20480], 20480)


def test_nsn_dq_workload_full_size_sampled():
    """The NSN workload (8 heads x 65536 tokens, b=2) through the double-quantized front end, keys per
    token and values in blocks of 32; sampled blocks against the oracle (pooled boundary rate), then
    decode by 32 query heads with one sampled KV head replaced by the oracle's own cache."""
    c = wl.NSN
    H, T, d, b = c["heads"], c["tokens"], c["d"], c["b"]
    hs = 5
    k = oracle.make_constants(d, b, c["handle_seed"])
    X = wl.nsn_tokens(H, T, d, c["seed"], device="cuda")
    Y = wl.nsn_tokens(H, T, d, c["seed"] + 1, device="cuda")
    with kvq.Handle(d, b, c["handle_seed"], qjl=False) as h:
        kc, kn, ks = run_dq(h, X)
        vc, vn, vs = run_dq(h, Y, layout=kvq.KVQ_LAYOUT_BLOCK32)
        rng = np.random.default_rng(13)
        for _ in range(24):
            hh, blk = int(rng.integers(H)), int(rng.integers(T // 128))
            sl = slice(blk * 128, (blk + 1) * 128)
            check_dq_head(k, X[hh, sl].double().cpu().numpy(), to_np_u32(kc[hh, sl]), to_np_f16bits(kn[hh, sl]),
                          ks[hh, blk:blk + 1].cpu().numpy(), pool="nsn_dq")
        Xs = X[hs].double().cpu().numpy()
        Ys = Y[hs].double().cpu().numpy()
        rk, wk, sk = _dq_oracle_stream(k, Xs)
        rv, wv, sv = _dq_oracle_stream(k, Ys)
        kc[hs] = torch.from_numpy(oracle.pack_codes(rk["codes"], b).view(np.int32)).cuda().reshape(T, b, d // 32)
        vc[hs] = torch.from_numpy(oracle.pack_codes_block32(rv["codes"], b).view(np.int32).reshape(T // 32, b, d)).cuda()
        kn[hs] = torch.from_numpy(wk).cuda()
        vn[hs] = torch.from_numpy(wv).cuda()
        ks[hs] = torch.from_numpy(rk["side"]).cuda()
        vs[hs] = torch.from_numpy(rv["side"]).cuda()
        q = wl.queries(1, 4 * H, d, seed=78, device="cuda")
        out = torch.empty((1, 4 * H, d), dtype=torch.float32, device="cuda")
        ws = torch.empty(kvq.kvq_decode_workspace(h, 1, 4 * H, H, T), dtype=torch.uint8, device="cuda")
        sl = torch.tensor([T], dtype=torch.int32, device="cuda")
        kvq.kvq_nsn_dq_decode_attend(h, q, H, kvq.make_cache(kc, None, kn, T, 0), kvq.make_cache(vc, None, vn, T, 1),
                                     ks, vs, sl, T, d ** -0.5, out, ws)
        assert kvq.kvq_status(h)[0] == 0
    qd = q.double().cpu().numpy()
    _, orf = oracle.nsn_dq_decode_attend(k, qd[0, 4 * hs:4 * hs + 4], sk, sv, rk["side"], rv["side"], d ** -0.5,
                                         want_logits=False)
    assert_close(out.cpu().numpy()[0, 4 * hs:4 * hs + 4], orf, "nsn-dq out (sampled head)")
    print("nsn_dq", pooled_check("nsn_dq"))


def test_window_over_a_double_quantized_cache_matches_oracle():
    """kvq_decode_attend_ex over an oracle-built double-quantized cache (ragged contexts) followed by fp16
    windows of different lengths: one softmax over the packed then the window tokens."""
    d, b, batch, hq, hkv, cap, wcap = 128, 2, 2, 8, 2, 512, 96
    seq_len, win_len = [384, 200], [77, 0]
    k = oracle.make_constants(d, b, 6)
    G, S = hq // hkv, batch * hkv
    R = oracle.nsn_dq_rec_bytes(d)
    kc = torch.zeros((S, cap, b, d // 32), dtype=torch.int32)
    vc = torch.zeros((S, cap // 32, b, d), dtype=torch.int32)
    kn = torch.zeros((S, cap), dtype=torch.float16)
    vn = torch.zeros_like(kn)
    ks = torch.zeros((S, cap // 128, R), dtype=torch.uint8)
    vs = torch.zeros_like(ks)
    st = []
    for s in range(S):
        rk, wk, sk = _dq_oracle_stream(k, wl.nsn_tokens(1, cap, d, seed=1100 + s)[0].double().numpy())
        rv, wv, sv = _dq_oracle_stream(k, wl.nsn_tokens(1, cap, d, seed=1200 + s)[0].double().numpy())
        kc[s] = torch.from_numpy(oracle.pack_codes(rk["codes"], b).view(np.int32))
        vc[s] = torch.from_numpy(oracle.pack_codes_block32(rv["codes"], b).view(np.int32).reshape(cap // 32, b, d))
        kn[s], vn[s] = torch.from_numpy(wk), torch.from_numpy(wv)
        ks[s], vs[s] = torch.from_numpy(rk["side"]), torch.from_numpy(rv["side"])
        st.append((sk, sv, rk["side"], rv["side"]))
    kw = wl.nsn_tokens(S, wcap, d, seed=1300).to(torch.float16)
    vw = wl.nsn_tokens(S, wcap, d, seed=1301).to(torch.float16)
    q = wl.queries(batch, hq, d, seed=83)
    max_T = max(seq_len)
    with kvq.Handle(d, b, 6, qjl=False) as h:
        out = torch.empty((batch, hq, d), dtype=torch.float32, device="cuda")
        logits = torch.empty((batch, hq, max_T + wcap), dtype=torch.float32, device="cuda")
        ws = torch.empty(kvq.kvq_decode_workspace(h, batch, hq, hkv, max_T), dtype=torch.uint8, device="cuda")
        kcd, vcd, knd, vnd, ksd, vsd = (t.cuda() for t in (kc, vc, kn, vn, ks, vs))
        kvq.kvq_decode_attend_ex(h, q.cuda(), hkv, kvq.make_cache(kcd, None, knd, cap, 0),
                                 kvq.make_cache(vcd, None, vnd, cap, 1),
                                 torch.tensor(seq_len, dtype=torch.int32, device="cuda"), max_T, d ** -0.5, out, ws,
                                 k_window=kw.cuda(), v_window=vw.cuda(),
                                 window_len=torch.tensor(win_len, dtype=torch.int32, device="cuda"),
                                 logits=logits, k_side=ksd, v_side=vsd)
        assert kvq.kvq_status(h)[0] == 0
        # side records and block means together are refused
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_decode_attend_ex(h, q.cuda(), hkv, kvq.make_cache(kcd, None, knd, cap, 0),
                                     kvq.make_cache(vcd, None, vnd, cap, 1),
                                     torch.tensor(seq_len, dtype=torch.int32, device="cuda"), max_T, d ** -0.5, out,
                                     ws, k_block_mean=torch.zeros((S, cap // 128, d), dtype=torch.float16,
                                                                  device="cuda"),
                                     v_block_mean=torch.zeros((S, cap // 128, d), dtype=torch.float16, device="cuda"),
                                     k_side=ksd, v_side=vsd)
        assert e.value.code == kvq.KVQ_EINVAL
        out, logits = out.cpu().numpy(), logits.cpu().numpy()
    qd = q.double().numpy()
    for bi in range(batch):
        T, W = seq_len[bi], win_len[bi]
        for hk in range(hkv):
            s = bi * hkv + hk
            sk, sv, rks, rvs = st[s]
            sk = {key: v[:T] for key, v in sk.items()}
            sv = {key: v[:T] for key, v in sv.items()}
            lr, orf = oracle.window_decode_attend(k, qd[bi, hk * G:(hk + 1) * G], sk, sv,
                                                  kw[s, :W].double().numpy(), vw[s, :W].double().numpy(), d ** -0.5,
                                                  False, dq=(rks, rvs))
            assert_close(out[bi, hk * G:(hk + 1) * G], orf, f"dq + window out b{bi} kvh{hk}")
            assert_close(logits[bi, hk * G:(hk + 1) * G, :T], lr[:, :T], f"dq + window packed logits b{bi} kvh{hk}")
            if W:
                assert_close(logits[bi, hk * G:(hk + 1) * G, max_T:max_T + W], lr[:, T:],
                             f"dq + window window logits b{bi} kvh{hk}")
