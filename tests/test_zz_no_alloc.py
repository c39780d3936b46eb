"""The decode entry point that allocates nothing, against the one that takes a workspace.

kvq_decode_attend_noalloc serves callers that cannot allocate device memory
when they decode (a fixed memory pool carved out at start-up, a plug-in
inside a runtime that owns every allocation).  It uses a scratch array
compiled into the library instead of a caller workspace.  This file runs
last so that a failure here never hides another test's result, and it must
pass both alone in a fresh process and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

from calibration_free_rotated_token_b200 import _abi as kvq
from calibration_free_rotated_token_b200 import workloads as wl

from .parity import ATOL, RTOL

pytestmark = pytest.mark.gpu


def _cache(h, S, T, seed, layout):
    """S streams of T quantized tokens of the Llama-layer key generator, on the device."""
    x = wl.llama_keys(S, T, h.d, seed, device="cuda")
    parts = [kvq.alloc_packed(h, T, layout=layout) for _ in range(S)]
    for s in range(S):
        kvq.kvq_quantize(h, x[s], *parts[s], layout=layout)
    return [torch.stack([p[i] for p in parts]) if parts[0][i] is not None else None for i in range(3)]


@pytest.mark.parametrize("b,qjl,Ts", [
    (2, True, (3008, 3008)),   # tensor-core path, the same sizes twice
    (2, True, (3008, 1056)),   # tensor-core path, fewer splits on the second call
    (4, True, (3008, 1056)),   # CUDA-core path (its own carving of the scratch), fewer splits next
    (3, False, (640, 2048)),   # 3-bit tensor-core path without QJL, more splits next
])
def test_noalloc_matches_workspace_entry_point_on_two_calls(b, qjl, Ts):
    """Two calls in a row, each against kvq_decode_attend on the same inputs; when the second
    call's context is shorter, nothing it reads may come from the first call's leftovers."""
    d, B, hq, hkv = 128, 2, 8, 2
    cap = max(Ts)
    with kvq.Handle(d, b, 1, qjl=qjl) as h:
        kt = _cache(h, B * hkv, cap, seed=5, layout=0)
        vt = _cache(h, B * hkv, cap, seed=6, layout=1)
        kc = kvq.make_cache(*kt, cap, 0)
        vc = kvq.make_cache(*vt, cap, 1)
        for call, T in enumerate(Ts):
            seq = torch.tensor([T, min(1777, T - 33)], dtype=torch.int32, device="cuda")
            ws = torch.empty(kvq.kvq_decode_workspace(h, B, hq, hkv, T), dtype=torch.uint8, device="cuda")
            assert ws.numel() <= kvq.NOALLOC_SCRATCH_BYTES
            q = wl.queries(B, hq, d, seed=100 + call, device="cuda")
            ref = torch.empty((B, hq, d), dtype=torch.float32, device="cuda")
            ref_l = torch.empty((B, hq, T), dtype=torch.float32, device="cuda")
            kvq.kvq_decode_attend(h, q, hkv, kc, vc, seq, T, d ** -0.5, ref, ws, ref_l)
            out = torch.full((B, hq, d), float("nan"), dtype=torch.float32, device="cuda")
            lg = torch.full((B, hq, T), float("nan"), dtype=torch.float32, device="cuda")
            kvq.kvq_decode_attend_noalloc(h, q, hkv, kc, vc, seq, T, d ** -0.5, out, lg)
            code, bits = kvq.kvq_status(h)
            assert code == 0, (code, bits)
            r, o = ref.cpu().numpy(), out.cpu().numpy()
            assert np.all(np.abs(o - r) <= ATOL + RTOL * np.abs(r)), f"call {call}: outputs differ"
            rl, ol = ref_l.cpu().numpy(), lg.cpu().numpy()
            fin = np.isfinite(rl)
            assert np.array_equal(fin, np.isfinite(ol))
            assert np.all(np.abs(ol[fin] - rl[fin]) <= ATOL + RTOL * np.abs(rl[fin])), f"call {call}: logits differ"


def test_noalloc_rejects_sizes_beyond_the_fixed_scratch():
    d, B, hq, hkv, T = 128, 64, 64, 8, 1 << 20
    with kvq.Handle(d, 2, 1, qjl=True) as h:
        assert kvq.kvq_decode_workspace(h, B, hq, hkv, T) > kvq.NOALLOC_SCRATCH_BYTES
        dummy = torch.zeros(64, dtype=torch.int32, device="cuda")
        kc = kvq.make_cache(dummy, dummy, dummy.view(torch.float16), T, 0)
        vc = kvq.make_cache(dummy, dummy, dummy.view(torch.float16), T, 1)
        q = torch.zeros((B, hq, d), dtype=torch.bfloat16, device="cuda")
        out = torch.empty((B, hq, d), dtype=torch.float32, device="cuda")
        seq = torch.zeros(B, dtype=torch.int32, device="cuda")
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_decode_attend_noalloc(h, q, hkv, kc, vc, seq, T, 1.0, out)
        assert e.value.code == kvq.KVQ_EINVAL and "scratch" in str(e.value)
