"""Decode attention over a packed cache plus a full-precision residual window
(kvq_decode_attend_ex), against the oracle's window_decode_attend; and the
flush-append cycle that moves a full window into the packed cache."""
import numpy as np
import pytest
import torch

import oracle
from calibration_free_rotated_token_b200 import _abi as kvq
from calibration_free_rotated_token_b200 import workloads as wl

from .parity import assert_close, compare_quantize, oracle_cache, to_np_f16bits, to_np_u32
from .test_gpu_decode import constants, upload_streams

pytestmark = pytest.mark.gpu


def check_window_case(d, b, qjl, batch, hq, hkv, seq_len, win_len, cap, win_cap, seed=3):
    k = constants(d, b, seed)
    G = hq // hkv
    S = batch * hkv
    kcs, vcs, kst, vst = [], [], [], []
    for s in range(S):
        T = seq_len[s // hkv]
        K = wl.llama_keys(1, T, d, seed=1100 + s)[0].double().numpy()
        V = wl.llama_values(1, T, d, seed=1200 + s)[0].double().numpy()
        c, q, n, st = oracle_cache(k, K, qjl)
        kcs.append((c, q, n)); kst.append(st)
        c, q, n, st = oracle_cache(k, V, qjl, layout=1)
        vcs.append((c, q, n)); vst.append(st)
    kw = wl.llama_keys(S, win_cap, d, seed=1300).to(torch.float16)   # [S, win_cap, d]
    vw = wl.llama_values(S, win_cap, d, seed=1301).to(torch.float16)
    qv = wl.queries(batch, hq, d, seed=79)
    max_T = max(seq_len)
    scale = 1 / np.sqrt(d)
    with kvq.Handle(d, b, seed, qjl=qjl) as h:
        kc, _kt = upload_streams(h, kcs, cap, 0)
        vc, _vt = upload_streams(h, vcs, cap, 1)
        out = torch.empty((batch, hq, d), dtype=torch.float32, device="cuda")
        logits = torch.full((batch, hq, max_T + win_cap), 7.0, dtype=torch.float32, device="cuda")
        ws = torch.empty(kvq.kvq_decode_workspace(h, batch, hq, hkv, max_T), dtype=torch.uint8, device="cuda")
        kvq.kvq_decode_attend_ex(h, qv.cuda(), hkv, kc, vc, torch.tensor(seq_len, dtype=torch.int32, device="cuda"),
                                 max_T, scale, out, ws, k_window=kw.cuda(), v_window=vw.cuda(),
                                 window_len=torch.tensor(win_len, dtype=torch.int32, device="cuda"), logits=logits)
        code, bits = kvq.kvq_status(h)
        assert code == 0, (code, bits)
        out, logits = out.cpu().numpy(), logits.cpu().numpy()
    qd = qv.double().numpy()
    for bi in range(batch):
        T, W = seq_len[bi], win_len[bi]
        for hk in range(hkv):
            s = bi * hkv + hk
            lr, orf = oracle.window_decode_attend(k, qd[bi, hk * G:(hk + 1) * G], kst[s], vst[s],
                                                  kw[s, :W].double().numpy(), vw[s, :W].double().numpy(), scale, qjl)
            assert_close(out[bi, hk * G:(hk + 1) * G], orf, f"out b{bi} kvh{hk}")
            rows = logits[bi, hk * G:(hk + 1) * G]
            if T > 0:
                assert_close(rows[:, :T], lr[:, :T], f"packed logits b{bi} kvh{hk}")
            if W > 0:
                assert_close(rows[:, max_T:max_T + W], lr[:, T:], f"window logits b{bi} kvh{hk}")


@pytest.mark.parametrize("d,b,qjl,batch,hq,hkv,seq_len,win_len,cap,win_cap", [
    (128, 2, True, 2, 8, 2, [1000, 320], [17, 128], 1024, 128),    # tensor-core path, GQA 4:1
    (64, 1, False, 1, 4, 4, [640], [200], 640, 256),               # GQA 1:1, a long window
    (128, 3, True, 2, 4, 1, [513, 64], [0, 31], 544, 32),          # 3-bit path, an empty window
    (128, 2, False, 1, 16, 2, [900], [96], 928, 128),              # GQA 8:1
    (256, 2, True, 2, 4, 2, [0, 300], [40, 1], 320, 64),           # an empty packed cache
])
def test_window_decode_matches_oracle(d, b, qjl, batch, hq, hkv, seq_len, win_len, cap, win_cap):
    check_window_case(d, b, qjl, batch, hq, hkv, seq_len, win_len, cap, win_cap)


def test_window_rejects_bad_arguments():
    with kvq.Handle(128, 2, 1, qjl=True) as h:
        codes, qjl, norms = kvq.alloc_packed(h, 64)
        kc = kvq.make_cache(codes, qjl, norms, 64, 0)
        vcodes, vqjl, vnorms = kvq.alloc_packed(h, 64, layout=1)
        vc = kvq.make_cache(vcodes, vqjl, vnorms, 64, 1)
        q = torch.randn(1, 4, 128, device="cuda").bfloat16()
        out = torch.empty(1, 4, 128, device="cuda")
        ws = torch.empty(kvq.kvq_decode_workspace(h, 1, 4, 1, 64), dtype=torch.uint8, device="cuda")
        sl = torch.tensor([64], dtype=torch.int32, device="cuda")
        big = torch.zeros(1, 300, 128, dtype=torch.float16, device="cuda")
        with pytest.raises(kvq.KvqError):  # window_cap above KVQ_MAX_WINDOW
            kvq.kvq_decode_attend_ex(h, q, 1, kc, vc, sl, 64, 1.0, out, ws, k_window=big, v_window=big,
                                     window_len=torch.tensor([3], dtype=torch.int32, device="cuda"))
        with pytest.raises(ValueError):  # a window without its lengths
            kvq.kvq_decode_attend_ex(h, q, 1, kc, vc, sl, 64, 1.0, out, ws, k_window=big[:, :8], v_window=big[:, :8])
        with pytest.raises(kvq.KvqError):  # NSN block means on a QJL handle
            kvq.kvq_decode_attend_ex(h, q, 1, kc, vc, sl, 64, 1.0, out, ws,
                                     k_block_mean=torch.zeros(128, dtype=torch.float16, device="cuda"),
                                     v_block_mean=torch.zeros(128, dtype=torch.float16, device="cuda"))


def test_flush_append_cycle():
    """Tokens arrive one by one into a 32-token fp16 window; a full window is flushed by
    kvq_quantize_batch into the packed arrays at offset seq_len (keys per token, values in
    blocks of 32).  The incrementally built cache equals one quantize over all flushed tokens and
    matches the oracle's quantization of them; decoding the oracle's own cache of those tokens
    plus the live window then matches the oracle's window decode."""
    d, b, W, steps = 128, 2, 32, 203
    hkv, hq = 2, 8
    cap = 256
    X = wl.llama_keys(hkv, steps, d, seed=1400).cuda()      # [hkv, steps, d]
    Y = wl.llama_values(hkv, steps, d, seed=1401).cuda()
    k = constants(d, b, 4)
    with kvq.Handle(d, b, 4, qjl=True) as h:
        kcodes = torch.zeros((hkv, cap, b, d // 32), dtype=torch.int32, device="cuda")
        kqjl = torch.zeros((hkv, cap, d // 32), dtype=torch.int32, device="cuda")
        kn = torch.zeros((hkv, cap, 2), dtype=torch.float16, device="cuda")
        vcodes = torch.zeros((hkv, cap // 32, b, d), dtype=torch.int32, device="cuda")
        vqjl = torch.zeros((hkv, cap // 32, d), dtype=torch.int32, device="cuda")
        vn = torch.zeros_like(kn)
        kwin = torch.zeros((hkv, W, d), dtype=torch.float16, device="cuda")
        vwin = torch.zeros_like(kwin)
        T, n = 0, 0
        for t in range(steps):
            kwin[:, n] = X[:, t].half()
            vwin[:, n] = Y[:, t].half()
            n += 1
            if n == W:  # flush: the window's fp16 tokens into the packed cache at offset T
                jobs = []
                for s in range(hkv):
                    jobs.append((kwin[s], kcodes[s, T:T + W], kqjl[s, T:T + W], kn[s, T:T + W], 0))
                    jobs.append((vwin[s], vcodes[s, T // 32:(T + W) // 32], vqjl[s, T // 32:(T + W) // 32],
                                 vn[s, T:T + W], 1))
                kvq.kvq_quantize_batch(h, jobs)
                T += W
                n = 0
        assert kvq.kvq_status(h)[0] == 0
        assert T == 192 and n == 11
        caches = []
        for s in range(hkv):
            Kf = X[s, :T].half()
            Vf = Y[s, :T].half()
            # the same tokens quantized at once
            c1, q1, n1 = kvq.alloc_packed(h, T)
            kvq.kvq_quantize(h, Kf, c1, q1, n1)
            assert torch.equal(c1.reshape(T, -1), kcodes[s, :T].reshape(T, -1))
            assert torch.equal(q1.reshape(T, -1), kqjl[s, :T].reshape(T, -1)) and torch.equal(n1, kn[s, :T])
            # the flushed records against the oracle's quantization of the same fp16 tokens
            Kd, Vd = Kf.double().cpu().numpy(), Vf.double().cpu().numpy()
            compare_quantize(k, Kd, to_np_u32(kcodes[s, :T]), to_np_u32(kqjl[s, :T]), to_np_f16bits(kn[s, :T]), True)
            compare_quantize(k, Vd, to_np_u32(vcodes[s, :T // 32]), to_np_u32(vqjl[s, :T // 32]),
                             to_np_f16bits(vn[s, :T]), True, layout=1)
            caches.append((oracle_cache(k, Kd, True), oracle_cache(k, Vd, True, layout=1)))
        # decode the oracle's own cache of the flushed tokens, plus the live window
        kc_, _kt = upload_streams(h, [c[0][:3] for c in caches], cap, 0)
        vc_, _vt = upload_streams(h, [c[1][:3] for c in caches], cap, 1)
        q = wl.queries(1, hq, d, seed=80, device="cuda")
        out = torch.empty((1, hq, d), dtype=torch.float32, device="cuda")
        ws = torch.empty(kvq.kvq_decode_workspace(h, 1, hq, hkv, cap), dtype=torch.uint8, device="cuda")
        kvq.kvq_decode_attend_ex(h, q, hkv, kc_, vc_, torch.tensor([T], dtype=torch.int32, device="cuda"), cap,
                                 1 / np.sqrt(d), out, ws, k_window=kwin, v_window=vwin,
                                 window_len=torch.tensor([n], dtype=torch.int32, device="cuda"))
        assert kvq.kvq_status(h)[0] == 0
    G = hq // hkv
    qd = q.double().cpu().numpy()
    out = out.cpu().numpy()
    for s in range(hkv):
        kst, vst = caches[s][0][3], caches[s][1][3]
        _, orf = oracle.window_decode_attend(k, qd[0, s * G:(s + 1) * G], kst, vst, kwin[s, :n].double().cpu().numpy(),
                                             vwin[s, :n].double().cpu().numpy(), 1 / np.sqrt(d), True)
        assert_close(out[0, s * G:(s + 1) * G], orf, f"out kvh{s}")


def test_window_over_nsn_cache_matches_oracle():
    """An NSN cache (oracle-built) followed by a 128-token fp16 window: the window's value sum
    enters the block-mean slot of its partial."""
    from .test_gpu_nsn import _nsn_oracle_stream
    d, b, hkv, hq, cap, T, W = 128, 2, 2, 8, 512, 384, 77
    k = oracle.make_constants(d, b, 5)
    G = hq // hkv
    kc = torch.zeros((hkv, cap, b, d // 32), dtype=torch.int32)
    vc = torch.zeros((hkv, cap // 32, b, d), dtype=torch.int32)
    kn = torch.zeros((hkv, cap, 2), dtype=torch.float16)
    vn = torch.zeros_like(kn)
    km = torch.zeros((hkv, cap // 128, d), dtype=torch.float16)
    vm = torch.zeros_like(km)
    st = []
    for s in range(hkv):
        rk, nbk, sk = _nsn_oracle_stream(k, wl.nsn_tokens(1, cap, d, seed=1500 + s)[0].double().numpy())
        rv, nbv, sv = _nsn_oracle_stream(k, wl.nsn_tokens(1, cap, d, seed=1600 + s)[0].double().numpy())
        kc[s] = torch.from_numpy(oracle.pack_codes(rk["codes"], b).view(np.int32))
        vc[s] = torch.from_numpy(oracle.pack_codes_block32(rv["codes"], b).view(np.int32).reshape(cap // 32, b, d))
        kn[s], vn[s] = torch.from_numpy(nbk), torch.from_numpy(nbv)
        km[s] = torch.from_numpy(rk["mean_half"].view(np.float16))
        vm[s] = torch.from_numpy(rv["mean_half"].view(np.float16))
        st.append((sk, sv, rk["mean_half"], rv["mean_half"]))
    kw = wl.nsn_tokens(hkv, 128, d, seed=1700).to(torch.float16)
    vw = wl.nsn_tokens(hkv, 128, d, seed=1701).to(torch.float16)
    q = wl.queries(1, hq, d, seed=81)
    with kvq.Handle(d, b, 5, qjl=False) as h:
        out = torch.empty((1, hq, d), dtype=torch.float32, device="cuda")
        ws = torch.empty(kvq.kvq_decode_workspace(h, 1, hq, hkv, cap), dtype=torch.uint8, device="cuda")
        kcd, vcd, knd, vnd, kmd, vmd = (t.cuda() for t in (kc, vc, kn, vn, km, vm))
        kvq.kvq_decode_attend_ex(h, q.cuda(), hkv, kvq.make_cache(kcd, None, knd, cap, 0),
                                 kvq.make_cache(vcd, None, vnd, cap, 1),
                                 torch.tensor([T], dtype=torch.int32, device="cuda"), cap, d ** -0.5, out, ws,
                                 k_window=kw.cuda(), v_window=vw.cuda(),
                                 window_len=torch.tensor([W], dtype=torch.int32, device="cuda"),
                                 k_block_mean=kmd, v_block_mean=vmd)
        assert kvq.kvq_status(h)[0] == 0
        out = out.cpu().numpy()
    qd = q.double().numpy()
    for s in range(hkv):
        sk, sv, mk, mv = st[s]
        sk = {key: v[:T] for key, v in sk.items()}
        sv = {key: v[:T] for key, v in sv.items()}
        _, orf = oracle.window_decode_attend(k, qd[0, s * G:(s + 1) * G], sk, sv, kw[s, :W].double().numpy(),
                                             vw[s, :W].double().numpy(), d ** -0.5, False,
                                             nsn=(mk[:T // 128], mv[:T // 128]))
        assert_close(out[0, s * G:(s + 1) * G], orf, f"nsn + window out kvh{s}")
