"""Benchmark of the rotated-token KV-cache quantizer on B200.

Headline line: KV quantize tokens/s on one Llama-3-8B-shaped layer (8 KV
heads x 32768 tokens x head_dim 128, bf16 K and V, 2-bit Lloyd-Max codes +
1-bit QJL with m = 128).  One step quantizes that layer's K and V (two
launches of the quantize kernel); a token is one position of the layer
(8 heads x (K + V) = 16 vectors).  The same JSON line carries the measured
decode attention (batch 16, 32/8 heads, 131072-token packed contexts) in
GB/s of packed cache and the NSN front end (8 x 65536 x 128) in tokens/s.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch one process per GPU with torch.distributed.run; every rank
quantizes its own layer (weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV quantize tokens/s"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode-attention measurement")
    ap.add_argument("--no-nsn", action="store_true", help="skip the NSN front-end measurement")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-sweep", action="store_true", help="skip the bit-width / head-dim sweep")
    ap.add_argument("--cpu-vectors", type=int, default=163840, help="vectors in the CPU oracle sample")
    ap.add_argument("--only", choices=("quantize", "decode", "nsn", "sweep"), default=None,
                    help="run one part only (for profiler captures); prints that part's result")
    ap.add_argument("--decode-T", type=int, default=None,
                    help="context length of the decode measurement (default: the workload's 131072)")
    ap.add_argument("--soak", type=float, default=1.5,
                    help="seconds of untimed steps under the clock sampler before the timed region")
    ap.add_argument("--sweep-rows", default=None,
                    help="run only these sweep rows, as d:b:qjl[,d:b:qjl...] (qjl 0 or 1; for profiler captures)")
    return ap.parse_args()


# ----------------------------------------------------------------------------
# plumbing
# ----------------------------------------------------------------------------
class Dist:
    """One process per GPU (torchrun env).  Only a barrier and a max-reduction of
    timings cross ranks: each rank works on its own layer / sequences.  The
    backend is NCCL on the GPUs ("gloo" on CPU for the multi-rank host tests)."""

    def __init__(self, n_gpus: int, backend: str = "nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if self.world != n_gpus:
            raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={self.world}")
        self.pg = None
        self.dev = torch.device("cuda", self.local) if backend == "nccl" else torch.device("cpu")
        if self.world > 1:
            import datetime

            import torch.distributed as dist

            kw = {}
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = self.dev
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=self.dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def whole_job_rate(world: int, units_per_rank: float, ms_max: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank / (ms_max / 1e3)


def tensor_record(n: int, d: int, launch_s: float) -> dict:
    """Algorithmic tensor-core throughput of one quantize launch: the S r
    projection (2 m d flop per vector, m = d) and the Hadamard rotation (2 d^2)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    peak, src = 1590.0, "fallback"
    if os.path.exists(p):
        with open(p) as f:
            peak, src = float(json.load(f)["bf16_tflops"]), "measured"
    sr = 2.0 * d * d * n / launch_s / 1e12
    rot = 2.0 * d * d * n / launch_s / 1e12
    return {"sr_projection_tflops": round(sr, 1), "rotation_tflops": round(rot, 1),
            "peak_bf16_tflops": peak, "peak_source": src, "frac": round((sr + rot) / peak, 4),
            "note": "fp16 S r (one fp16 residual term) and bf16 x (H D)^T, fp32 accumulate; "
                    "the S r contraction is the method's, the rotation is this kernel's choice"}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class Clocks:
    """nvidia-smi samples of the current GPU during a timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.rows = []
        if self.proc is None:
            return
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        for r in csv.reader(io.StringIO(out)):
            if len(r) >= 9:
                self.rows.append([c.strip() for c in r])

    def summary(self):
        rows = getattr(self, "rows", [])
        if not rows:
            return None
        def num(s):
            try:
                return float(s)
            except ValueError:
                return float("nan")
        sm = [num(r[1]) for r in rows]
        mx = max(num(r[2]) for r in rows)
        loaded = [s for s in sm if s == s and s > 0.5 * mx] or sm
        reasons = set()
        for r in rows:
            for name, col in (("hw_slowdown", 5), ("hw_thermal_slowdown", 6), ("sw_thermal_slowdown", 7),
                              ("sw_power_cap", 8)):
                if r[col].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(rows), "power_w_max": max(num(r[3]) for r in rows)}


HEAD_START_CYCLES = 6_000_000  # ~3 ms at 1.97 GHz


def timed(dist: Dist, fn, steps: int, stream) -> float:
    """Milliseconds for `steps` calls of fn(i), device-timed, max over ranks."""
    dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    # A device-side sleep ahead of the region lets the host enqueue the steps
    # before the GPU reaches them, so the device intervals hold no host
    # launch latency (that is what the e2e figure measures).
    torch.cuda._sleep(HEAD_START_CYCLES)
    e0.record(stream)
    for i in range(steps):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    return dist.max(e0.elapsed_time(e1))


_L2_FLUSH = None


def timed_flushed(dist: Dist, fn, steps: int, stream) -> float:
    """Milliseconds for `steps` calls of fn(i) whose data would fit in L2: each
    call is timed alone on the device, after a 256 MB write (twice the L2) has
    evicted the previous call's data; the sum over the calls, max over ranks."""
    global _L2_FLUSH
    if _L2_FLUSH is None:
        _L2_FLUSH = torch.empty(64 << 20, dtype=torch.int32, device="cuda")
    dist.barrier()
    torch.cuda.synchronize()
    evs = []
    with torch.cuda.stream(stream):
        for i in range(steps):
            _L2_FLUSH.fill_(i)
            # as in timed(): the host enqueues the call before the device reaches it
            torch.cuda._sleep(HEAD_START_CYCLES // 8)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn(i)
            e1.record(stream)
            evs.append((e0, e1))
    torch.cuda.synchronize()
    dist.barrier()
    return dist.max(sum(a.elapsed_time(b) for a, b in evs))


def traffic_record(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current build."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    fp = os.path.join(ROOT, "_build", "libkvq.fingerprint")
    if not (os.path.exists(p) and os.path.exists(fp)):
        return None
    with open(p) as f:
        j = json.load(f)
    rec = j.get(kernel)
    if not rec or rec.get("fingerprint") != open(fp).read().strip():
        return None
    return rec.get("dram_bytes_per_launch")


def parity_record():
    """Boundary-excluded code counts per workload, pooled by the parity tests
    (tests/test_gpu_boundary_rates.py, written with KVQ_PARITY_RECORD) and
    committed under profiles/; null when absent."""
    p = os.path.join(ROOT, "profiles", "parity_boundary.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    return {"bar": j.get("bar"), "source": "profiles/parity_boundary.json",
            "workloads": {k: {"excluded": v["excluded"], "coords": v["coords"], "rate": float(f"{v['rate']:.3g}")}
                          for k, v in j.get("workloads", {}).items()}}


# ----------------------------------------------------------------------------
# our implementation
# ----------------------------------------------------------------------------
def bench_quantize(args, dist):
    from calibration_free_rotated_token_b200 import _abi as kvq
    from calibration_free_rotated_token_b200 import workloads as wl

    c = wl.LLAMA_LAYER
    H, T, d, b = c["heads"], c["tokens"], c["d"], c["b"]
    h = kvq.Handle(d, b, c["handle_seed"], qjl=True)
    copies = []
    for i in range(4):
        K = wl.llama_keys(H, T, d, c["k_seed"] + 100 * i + 1000 * dist.rank, device="cuda").reshape(-1, d)
        V = wl.llama_values(H, T, d, c["v_seed"] + 100 * i + 1000 * dist.rank, device="cuda").reshape(-1, d)
        copies.append((K, V))
    n = H * T
    outK = kvq.alloc_packed(h, n)                                  # keys: one record per token
    outV = kvq.alloc_packed(h, n, layout=kvq.KVQ_LAYOUT_BLOCK32)    # values: blocks of 32 tokens
    stream = torch.cuda.current_stream()

    def step(i):
        # keys and values of the layer in one launch (two streams of vectors)
        K, V = copies[i % 4]
        kvq.kvq_quantize_batch(h, [(K, *outK, kvq.KVQ_LAYOUT_TOKEN), (V, *outV, kvq.KVQ_LAYOUT_BLOCK32)],
                               stream=stream)

    for i in range(args.warmup):
        step(i)
    code, bits = kvq.kvq_status(h)
    if code != 0:
        raise RuntimeError(f"quantize status {code} bits {bits}")
    # The K-step region lasts milliseconds, shorter than the sampler's period:
    # the sampler runs over an untimed soak of the same step and the region.
    with Clocks(torch.cuda.current_device()) as clk:
        t_end = time.time() + args.soak
        i = 0
        while time.time() < t_end:
            step(i)
            i += 1
            if i % 64 == 0:
                torch.cuda.synchronize()
        ms = timed(dist, step, args.steps, stream)
    code, bits = kvq.kvq_status(h)
    if code != 0:
        raise RuntimeError(f"quantize status {code} bits {bits}")

    bytes_per_vec = 2 * d + b * d // 8 + d // 8 + 4
    per_launch_bytes = 2 * n * bytes_per_vec  # one launch quantizes the layer's K and V
    # The timed region holds nothing but the quantize launches (one per step,
    # back to back on one stream, so each next launch's set-up overlaps the
    # previous one's tail): the average launch is the region over the launches.
    avg_launch_s = ms / args.steps / 1e3
    hbm, src = peaks()
    achieved = per_launch_bytes / avg_launch_s / 1e9
    res = dict(ms=ms, tokens_per_step=T, vectors_per_step=2 * n, launches=args.steps,
               roofline={"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(achieved / hbm, 4), "traffic": traffic_record("quantize_llama_layer"),
                         "peak_source": f"{src} hbm_gbs (copy)",
                         "kernel": "quantize_tc_kernel<128,2,qjl,bf16> (K and V of the layer in one launch)",
                         "algorithmic_bytes_per_launch": per_launch_bytes,
                         "avg_launch_ms": round(avg_launch_s * 1e3, 5),
                         "frac_of_spec_8tbs": round(achieved / SPEC_HBM_GBS, 4)},
               tensor=tensor_record(2 * n, d, avg_launch_s),
               clocks=clk.summary())

    # ---- the same step with the rotation on the CUDA cores: the in-register
    # transform kernel (one launch for K, one for V), for comparison ----
    hc = kvq.Handle(d, b, c["handle_seed"], qjl=True, cuda_core_rotation=True)

    def step_cc(i):
        K, V = copies[i % 4]
        kvq.kvq_quantize_batch(hc, [(K, *outK, kvq.KVQ_LAYOUT_TOKEN), (V, *outV, kvq.KVQ_LAYOUT_BLOCK32)],
                               stream=stream)

    for i in range(args.warmup):
        step_cc(i)
    ms_cc = timed(dist, step_cc, args.steps, stream)
    code, bits = kvq.kvq_status(hc)
    if code != 0:
        raise RuntimeError(f"quantize (CUDA-core rotation) status {code} bits {bits}")
    hc.close()
    cc_s = ms_cc / args.steps / 1e3
    res["rotation"] = {
        "tensor_core_us_per_step": round(avg_launch_s * 1e6, 2),
        "cuda_core_us_per_step": round(cc_s * 1e6, 2),
        "cuda_core_gbs": round(per_launch_bytes / cc_s / 1e9, 1),
        "cuda_core_frac_of_hbm": round(per_launch_bytes / cc_s / 1e9 / hbm, 4),
        "speedup_of_tensor_core_rotation": round(cc_s / avg_launch_s, 3),
        "note": "the same layer step (K and V, same outputs under the same parity rules) with KVQ_CUDA_CORE_ROTATION: "
                "quantize_kernel with the in-register Walsh-Hadamard transform, one launch per job"}

    # ---- end to end through the binding with host buffers ----
    # Every step copies its K and V from pinned host memory, quantizes them
    # through the C ABI and copies the codes, QJL bits and norms back.  As a
    # user streaming layers would, the steps are double-buffered on three
    # streams: step i+1's upload, step i's quantize and step i-1's download
    # overlap (PCIe is full duplex); events order each buffer's reuse.
    Kh = copies[0][0].cpu().pin_memory()
    Vh = copies[0][1].cpu().pin_memory()
    Kd = [torch.empty_like(copies[0][0]) for _ in range(2)]
    Vd = [torch.empty_like(copies[0][1]) for _ in range(2)]
    outs = [(outK, outV), (kvq.alloc_packed(h, n), kvq.alloc_packed(h, n, layout=kvq.KVQ_LAYOUT_BLOCK32))]
    host_out = [[[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in o] for o in slot] for slot in outs]
    s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_done + ev_out:
        e.record(stream)

    def e2e_step(i):
        sl = i % 2
        with torch.cuda.stream(s_up):
            s_up.wait_event(ev_done[sl])  # step i-2's quantize has read this input buffer
            Kd[sl].copy_(Kh, non_blocking=True)
            Vd[sl].copy_(Vh, non_blocking=True)
            ev_in[sl].record(s_up)
        stream.wait_event(ev_in[sl])
        stream.wait_event(ev_out[sl])  # step i-2's download has read this output buffer
        oK, oV = outs[sl]
        kvq.kvq_quantize_batch(h, [(Kd[sl], *oK, kvq.KVQ_LAYOUT_TOKEN), (Vd[sl], *oV, kvq.KVQ_LAYOUT_BLOCK32)],
                               stream=stream)
        ev_done[sl].record(stream)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev_done[sl])
            for ho, do in zip(host_out[sl], outs[sl]):
                for x, y in zip(ho, do):
                    x.copy_(y, non_blocking=True)
            ev_out[sl].record(s_down)

    def e2e_timed(steps):
        dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(HEAD_START_CYCLES)  # on `stream`; the uploads wait for it through e0
        e0.record(stream)
        s_up.wait_event(e0)
        for i in range(steps):
            e2e_step(i)
        stream.wait_event(ev_out[(steps - 1) % 2])
        stream.wait_event(ev_out[steps % 2])
        e1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        return dist.max(e0.elapsed_time(e1))

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    e2e_steps = max(8, args.steps)
    ms_e2e = e2e_timed(e2e_steps)
    h2d = Kh.numel() * Kh.element_size() + Vh.numel() * Vh.element_size()
    d2h = sum(t.numel() * t.element_size() for o in host_out[0] for t in o)
    res["e2e"] = {"value": dist.world * T * e2e_steps / (ms_e2e / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                  "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e / e2e_steps,
                  "path": "pinned host K,V -> kvq_quantize_batch (C ABI) -> pinned host codes, qjl, norms; "
                          "double-buffered on three streams (step i+1's upload, step i's quantize and step "
                          "i-1's download overlap)"}
    rows = min(max(args.cpu_vectors, 24576 * (os.cpu_count() or 1)) // 2, n)  # enough for the sharded oracle run
    res["sample_input"] = (copies[0][0][:rows].cpu(), copies[0][1][:rows].cpu())
    h.close()
    return res


def bench_decode(args, dist):
    from calibration_free_rotated_token_b200 import _abi as kvq
    from calibration_free_rotated_token_b200 import workloads as wl

    c = wl.DECODE
    B, hq, hkv, d, T = c["batch"], c["hq"], c["hkv"], c["d"], (args.decode_T or c["T"])
    h = kvq.Handle(d, c["b"], c["handle_seed"], qjl=True)
    S = B * hkv
    kc = torch.empty((S, T, h.b, d // 32), dtype=torch.int32, device="cuda")
    vc = torch.empty((S, T // 32, h.b, d), dtype=torch.int32, device="cuda")
    kq = torch.empty((S, T, d // 32), dtype=torch.int32, device="cuda")
    vq = torch.empty((S, T // 32, d), dtype=torch.int32, device="cuda")
    kn = torch.empty((S, T, 2), dtype=torch.float16, device="cuda")
    vn = torch.empty_like(kn)
    for bi in range(B):
        sl = slice(bi * hkv, (bi + 1) * hkv)
        K = wl.llama_keys(hkv, T, d, wl.cache_slice_seed(c["handle_seed"], bi, dist.rank, 0), device="cuda")
        kvq.kvq_quantize(h, K, kc[sl], kq[sl], kn[sl])
        del K
        V = wl.llama_values(hkv, T, d, wl.cache_slice_seed(c["handle_seed"], bi, dist.rank, 1), device="cuda")
        for hk in range(hkv):
            s_ = bi * hkv + hk
            kvq.kvq_quantize(h, V[hk], vc[s_], vq[s_], vn[s_], layout=kvq.KVQ_LAYOUT_BLOCK32)
        del V
    q = wl.queries(B, hq, d, c["q_seed"], device="cuda", std=c["q_std"])
    out = torch.empty((B, hq, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(kvq.kvq_decode_workspace(h, B, hq, hkv, T), dtype=torch.uint8, device="cuda")
    seq = torch.full((B,), T, dtype=torch.int32, device="cuda")
    kcache = kvq.make_cache(kc, kq, kn, T, kvq.KVQ_LAYOUT_TOKEN)
    vcache = kvq.make_cache(vc, vq, vn, T, kvq.KVQ_LAYOUT_BLOCK32)
    stream = torch.cuda.current_stream()

    def step(i):
        kvq.kvq_decode_attend(h, q, hkv, kcache, vcache, seq, T, c["scale"], out, ws, stream=stream)

    for i in range(max(3, args.warmup)):
        step(i)
    code, bits = kvq.kvq_status(h)
    if code != 0:
        raise RuntimeError(f"decode status {code} bits {bits}")
    steps = max(5, args.steps // 2)
    ms = timed(dist, step, steps, stream)
    cache_bytes = S * T * 2 * (h.b * d // 8 + d // 8 + 4)
    gbs = cache_bytes / (ms / steps / 1e3) / 1e9
    hbm, src = peaks()

    # the same call with a 128-token fp16 residual window per (sequence, KV head)
    W = 128
    kw = wl.llama_keys(S, W, d, c["q_seed"] + 1, device="cuda").half()
    vw = wl.llama_values(S, W, d, c["q_seed"] + 2, device="cuda").half()
    wl_len = torch.full((B,), W, dtype=torch.int32, device="cuda")

    def wstep(i):
        kvq.kvq_decode_attend_ex(h, q, hkv, kcache, vcache, seq, T, c["scale"], out, ws, k_window=kw, v_window=vw,
                                 window_len=wl_len, stream=stream)

    for i in range(3):
        wstep(i)
    code, bits = kvq.kvq_status(h)
    if code != 0:
        raise RuntimeError(f"window decode status {code} bits {bits}")
    ms_w = timed(dist, wstep, steps, stream)
    h.close()
    return {"metric": "packed-cache decode-attn GB/s", "value": round(dist.world * gbs, 1), "unit": "GB/s",
            "frac_of_hbm": round(gbs / hbm, 4), "ms_per_step": ms / steps, "steps": steps,
            "workload": f"batch 16, 32 query / 8 KV heads, d 128, {T}-token contexts, b=2 + QJL, one bf16 query token",
            "cache_bytes_per_step": cache_bytes, "launches_per_step": 3,
            "with_window": {"window_tokens": W, "ms_per_step": ms_w / steps, "launches_per_step": 4,
                            "bytes_per_step": int(cache_bytes + S * W * d * 2 * 2),
                            "note": "kvq_decode_attend_ex: the packed cache plus a 128-token fp16 window per "
                                    "(sequence, KV head), attended exactly"},
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "frac_of_spec_8tbs": round(gbs / SPEC_HBM_GBS, 4),
                         "traffic": traffic_record("decode_split"),
                         "peak_source": f"{src} hbm_gbs (copy)",
                         "note": "whole decode call (qproj + split + combine); the split kernel dominates"}}


def bench_nsn(args, dist):
    from calibration_free_rotated_token_b200 import _abi as kvq
    from calibration_free_rotated_token_b200 import workloads as wl

    c = wl.NSN
    H, T, d = c["heads"], c["tokens"], c["d"]
    h = kvq.Handle(d, c["b"], c["handle_seed"], qjl=False)
    xs = [wl.nsn_tokens(H, T, d, c["seed"] + i + 1000 * dist.rank, device="cuda") for i in range(4)]
    codes = torch.empty((H, T, h.b, d // 32), dtype=torch.int32, device="cuda")
    norms = torch.empty((H, T, 2), dtype=torch.float16, device="cuda")
    means = torch.empty((H, T // 128, d), dtype=torch.float16, device="cuda")
    stream = torch.cuda.current_stream()

    def step(i):
        kvq.kvq_nsn_quantize(h, xs[i % 4], codes, norms, means, stream=stream)

    for i in range(max(3, args.warmup)):
        step(i)
    code, bits = kvq.kvq_status(h)
    if code != 0:
        raise RuntimeError(f"nsn status {code} bits {bits}")
    steps = args.steps
    ms = timed(dist, step, steps, stream)
    bytes_per_vec = 2 * d + h.b * d // 8 + 4 + 2 * d / 128
    gbs = H * T * bytes_per_vec / (ms / steps / 1e3) / 1e9
    hbm, src = peaks()
    del xs, codes, norms, means

    # ---- decode attention over NSN caches: 4 sequences of this workload (keys per token,
    # values in blocks of 32), 32 query heads on the 8 KV heads, one bf16 query token ----
    NB, hq = 4, 4 * H
    kc = torch.empty((NB * H, T, h.b, d // 32), dtype=torch.int32, device="cuda")
    vc = torch.empty((NB * H, T // 32, h.b, d), dtype=torch.int32, device="cuda")
    kn = torch.empty((NB * H, T, 2), dtype=torch.float16, device="cuda")
    vn = torch.empty_like(kn)
    km = torch.empty((NB * H, T // 128, d), dtype=torch.float16, device="cuda")
    vm = torch.empty_like(km)
    for bi in range(NB):
        sl = slice(bi * H, (bi + 1) * H)
        X = wl.nsn_tokens(H, T, d, c["seed"] + 100 + 2 * bi + 1000 * dist.rank, device="cuda")
        kvq.kvq_nsn_quantize(h, X, kc[sl], kn[sl], km[sl], stream=stream)
        X = wl.nsn_tokens(H, T, d, c["seed"] + 101 + 2 * bi + 1000 * dist.rank, device="cuda")
        kvq.kvq_nsn_quantize(h, X, vc[sl], vn[sl], vm[sl], stream=stream, layout=kvq.KVQ_LAYOUT_BLOCK32)
        del X
    q = wl.queries(NB, hq, d, c["seed"] + 7, device="cuda", std=d ** -0.5)
    out = torch.empty((NB, hq, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(kvq.kvq_decode_workspace(h, NB, hq, H, T), dtype=torch.uint8, device="cuda")
    seq = torch.full((NB,), T, dtype=torch.int32, device="cuda")
    kcache = kvq.make_cache(kc, None, kn, T, kvq.KVQ_LAYOUT_TOKEN)
    vcache = kvq.make_cache(vc, None, vn, T, kvq.KVQ_LAYOUT_BLOCK32)

    def dstep(i):
        kvq.kvq_nsn_decode_attend(h, q, H, kcache, vcache, km, vm, seq, T, 1.0, out, ws, stream=stream)

    for i in range(3):
        dstep(i)
    code, bits = kvq.kvq_status(h)
    if code != 0:
        raise RuntimeError(f"nsn decode status {code} bits {bits}")
    dsteps = max(5, steps // 2)
    ms_d = timed_flushed(dist, dstep, dsteps, stream)
    cache_bytes = NB * H * T * 2 * (h.b * d // 8 + 4 + 2 * d / 128)
    dgbs = cache_bytes / (ms_d / dsteps / 1e3) / 1e9
    del kc, vc, kn, vn, km, vm

    # ---- the same with double-quantized side data (4-bit norm and mean codes, fp16 ||w||) ----
    R = kvq.kvq_nsn_dq_side_bytes(d)
    xs = [wl.nsn_tokens(H, T, d, c["seed"] + i + 1000 * dist.rank, device="cuda") for i in range(4)]
    codes = torch.empty((H, T, h.b, d // 32), dtype=torch.int32, device="cuda")
    wn = torch.empty((H, T), dtype=torch.float16, device="cuda")
    side = torch.empty((H, T // 128, R), dtype=torch.uint8, device="cuda")

    def qstep_dq(i):
        kvq.kvq_nsn_dq_quantize(h, xs[i % 4], codes, wn, side, stream=stream)

    for i in range(3):
        qstep_dq(i)
    ms_q = timed(dist, qstep_dq, steps, stream)
    q_bytes = H * T * (2 * d + h.b * d // 8 + 2) + H * (T // 128) * R
    q_gbs = q_bytes / (ms_q / steps / 1e3) / 1e9
    del xs, codes, wn, side
    kc = torch.empty((NB * H, T, h.b, d // 32), dtype=torch.int32, device="cuda")
    vc = torch.empty((NB * H, T // 32, h.b, d), dtype=torch.int32, device="cuda")
    kn = torch.empty((NB * H, T), dtype=torch.float16, device="cuda")
    vn = torch.empty_like(kn)
    ks = torch.empty((NB * H, T // 128, R), dtype=torch.uint8, device="cuda")
    vs = torch.empty_like(ks)
    for bi in range(NB):
        sl = slice(bi * H, (bi + 1) * H)
        X = wl.nsn_tokens(H, T, d, c["seed"] + 100 + 2 * bi + 1000 * dist.rank, device="cuda")
        kvq.kvq_nsn_dq_quantize(h, X, kc[sl], kn[sl], ks[sl], stream=stream)
        X = wl.nsn_tokens(H, T, d, c["seed"] + 101 + 2 * bi + 1000 * dist.rank, device="cuda")
        kvq.kvq_nsn_dq_quantize(h, X, vc[sl], vn[sl], vs[sl], stream=stream, layout=kvq.KVQ_LAYOUT_BLOCK32)
        del X
    kcache = kvq.make_cache(kc, None, kn, T, kvq.KVQ_LAYOUT_TOKEN)
    vcache = kvq.make_cache(vc, None, vn, T, kvq.KVQ_LAYOUT_BLOCK32)

    def dstep_dq(i):
        kvq.kvq_nsn_dq_decode_attend(h, q, H, kcache, vcache, ks, vs, seq, T, 1.0, out, ws, stream=stream)

    for i in range(3):
        dstep_dq(i)
    code, bits = kvq.kvq_status(h)
    if code != 0:
        raise RuntimeError(f"nsn dq status {code} bits {bits}")
    ms_dd = timed_flushed(dist, dstep_dq, dsteps, stream)
    dq_cache = NB * H * T * 2 * (h.b * d // 8 + 2) + NB * H * (T // 128) * 2 * R
    dq_dgbs = dq_cache / (ms_dd / dsteps / 1e3) / 1e9
    h.close()
    return {"metric": "NSN quantize tokens/s", "value": dist.world * T * steps / (ms / 1e3), "unit": "tokens/s",
            "ms_per_step": ms / steps, "workload": "8 heads x 65536 tokens x d128 bf16, b=2, no QJL",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "frac_of_spec_8tbs": round(gbs / SPEC_HBM_GBS, 4),
                         "traffic": traffic_record("nsn_quantize"),
                         "peak_source": f"{src} hbm_gbs (copy)"},
            "decode": {"metric": "NSN packed-cache decode-attn GB/s", "value": round(dist.world * dgbs, 1),
                       "unit": "GB/s", "frac_of_hbm": round(dgbs / hbm, 4), "ms_per_step": ms_d / dsteps,
                       "steps": dsteps, "cache_bytes_per_step": int(cache_bytes),
                       "l2": "each call timed alone after a 256 MB write evicts L2 (the cache is about L2's size)",
                       "workload": "4 sequences x 8 KV heads x 65536 tokens of the NSN workload (b=2, keys per "
                                   "token, values in blocks of 32, fp16 block means), 32 query heads, one bf16 "
                                   "query token, kvq_nsn_decode_attend"},
            "double_quantized": {
                "quantize_ms_per_step": ms_q / steps, "quantize_gbs": round(q_gbs, 1),
                "quantize_frac_of_hbm": round(q_gbs / hbm, 4), "quantize_bytes_per_step": int(q_bytes),
                "decode_gbs": round(dist.world * dq_dgbs, 1), "decode_frac_of_hbm": round(dq_dgbs / hbm, 4),
                "decode_ms_per_step": ms_dd / dsteps, "decode_cache_bytes_per_step": int(dq_cache),
                "side_bits_per_element": round((R / 128 + 2) * 8 / d, 4),
                "l2": "decode calls timed alone after a 256 MB write evicts L2",
                "workload": "the same NSN workload through kvq_nsn_dq_quantize (4-bit token-norm and block-mean "
                            "codes in one side record per 128 tokens, fp16 ||w||) and kvq_nsn_dq_decode_attend"}}


def bench_sweep(args, dist):
    """Bit-width / head-dim sweep: per (d, b, QJL), the quantize of 2^20 keys and
    2^20 values (bf16 N(0, 1), 1% of the tokens x10) and one decode over them as
    8 KV heads x 131072 tokens with one query per head (scale 1/sqrt(d))."""
    from calibration_free_rotated_token_b200 import _abi as kvq
    from calibration_free_rotated_token_b200 import workloads as wl

    c = wl.SWEEP
    n, hkv, T = c["n"], c["hkv"], c["T"]
    hbm, src = peaks()
    stream = torch.cuda.current_stream()
    steps = max(5, args.steps // 3)
    keep = None
    if args.sweep_rows:
        keep = {tuple(int(v) for v in r.split(":")) for r in args.sweep_rows.split(",")}
    rows = []
    for d in c["dims"]:
        if keep is not None and not any(k[0] == d for k in keep):
            continue
        X = [wl.sweep_tokens(n, d, c["seed"] + 2 * d + i + 1000 * dist.rank, device="cuda") for i in range(2)]
        q = wl.queries(1, hkv, d, c["seed"] + 7 * d, device="cuda")
        seq = torch.full((1,), T, dtype=torch.int32, device="cuda")
        out = torch.empty((1, hkv, d), dtype=torch.float32, device="cuda")
        for b in c["bits"]:
            for qjl in c["qjl"]:
                if keep is not None and (d, b, int(qjl)) not in keep:
                    continue
                h = kvq.Handle(d, b, c["handle_seed"], qjl=qjl)
                outK = kvq.alloc_packed(h, n)
                outV = kvq.alloc_packed(h, n, layout=kvq.KVQ_LAYOUT_BLOCK32)

                def qstep(i):
                    kvq.kvq_quantize_batch(h, [(X[0], *outK, kvq.KVQ_LAYOUT_TOKEN),
                                               (X[1], *outV, kvq.KVQ_LAYOUT_BLOCK32)], stream=stream)

                for i in range(3):
                    qstep(i)
                ms_q = timed(dist, qstep, steps, stream)
                kcache = kvq.make_cache(*outK, T, kvq.KVQ_LAYOUT_TOKEN)
                vcache = kvq.make_cache(*outV, T, kvq.KVQ_LAYOUT_BLOCK32)
                ws = torch.empty(kvq.kvq_decode_workspace(h, 1, hkv, hkv, T), dtype=torch.uint8, device="cuda")

                def dstep(i):
                    kvq.kvq_decode_attend(h, q, hkv, kcache, vcache, seq, T, d ** -0.5, out, ws, stream=stream)

                for i in range(3):
                    dstep(i)
                ms_d = timed_flushed(dist, dstep, steps, stream)
                code, bits = kvq.kvq_status(h)
                if code != 0:
                    raise RuntimeError(f"sweep d={d} b={b} qjl={qjl}: status {code} bits {bits}")
                rec = b * d // 8 + (d // 8 if qjl else 0) + 4  # packed bytes per vector
                q_gbs = n * (2 * d + rec) / (ms_q / (2 * steps) / 1e3) / 1e9
                d_gbs = 2 * n * rec / (ms_d / steps / 1e3) / 1e9
                rows.append({"d": d, "b": b, "qjl": qjl,
                             "quantize_us_per_2e20": round(ms_q / (2 * steps) * 1e3, 2),
                             "quantize_gbs": round(q_gbs, 1),
                             "quantize_frac": round(q_gbs / hbm, 4),
                             "quantize_kernel": "quantize_tc_kernel" if d <= 128 or not qjl else "quantize_kernel",
                             "decode_us": round(ms_d / steps * 1e3, 2), "decode_gbs": round(d_gbs, 1),
                             "decode_frac": round(d_gbs / hbm, 4),
                             "decode_kernel": ("decode_mma_kernel" if b <= 2 or (b == 3 and d <= 128)
                                               else "decode_split_kernel")})
                h.close()
                del outK, outV, kcache, vcache, ws
        del X
    return {"workload": "per (d, b, QJL): quantize 2^20 keys + 2^20 values (bf16 N(0,1), 1% of tokens x10; "
                        "keys per token, values in blocks of 32; one kvq_quantize_batch call), then one decode "
                        "over them: 8 KV heads x "
                        "131072 tokens, one bf16 query per head",
            "bytes": "quantize: 2d in + the packed record out per vector; decode: the K and V records read",
            "l2": "quantize: two 2^20-vector inputs per call (256 MB-1 GB); decode: each call timed alone after a "
                  "256 MB write evicts L2 (the caches, 28-109 MB, fit in it)",
            "peak": hbm, "peak_source": f"{src} hbm_gbs (copy)", "steps": steps, "rows": rows}


SPEC_HBM_GBS = 8000.0  # B200 HBM3e specification (DGX figure)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_quantize_sharded(k, X, qjl: bool, threads: int):
    """The oracle's quantize over row ranges of X on `threads` host threads
    (the C oracle runs with the interpreter lock released; no shared state)."""
    import concurrent.futures as cf

    import oracle

    chunks = [c for c in np.array_split(X, threads) if c.shape[0] > 0]
    with cf.ThreadPoolExecutor(max_workers=len(chunks)) as ex:
        list(ex.map(lambda c: oracle.quantize(k, c, qjl), chunks))
    return len(chunks)


def cpu_baseline(sample, n_vectors: int):
    """The oracle, as it stands, on a bounded sample of the same workload (rank 0, N = 1)."""
    import oracle
    from calibration_free_rotated_token_b200 import workloads as wl

    c = wl.LLAMA_LAYER
    k = oracle.make_constants(c["d"], c["b"], c["handle_seed"])
    K, V = sample
    Kd = K.double().numpy()[: n_vectors // 2]
    Vd = V.double().numpy()[: n_vectors // 2]
    # (i) one thread
    t0 = time.perf_counter()
    oracle.quantize(k, Kd, True)
    oracle.quantize(k, Vd, True)
    dt1 = time.perf_counter() - t0
    vec1 = Kd.shape[0] + Vd.shape[0]
    # (ii) sharded over every host core (token ranges, no shared state)
    cores = os.cpu_count() or 1
    nsh = min(max(n_vectors, 24576 * cores), 2 * K.shape[0])
    Ks = K.double().numpy()[: nsh // 2]
    Vs = V.double().numpy()[: nsh // 2]
    t0 = time.perf_counter()
    used = oracle_quantize_sharded(k, Ks, True, cores)
    oracle_quantize_sharded(k, Vs, True, cores)
    dts = time.perf_counter() - t0
    vecs = Ks.shape[0] + Vs.shape[0]
    return {"value": vecs / 16 / dts, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": f"{vecs} vectors ({vecs // 16} tokens) of the layer's K and V, fp64 C++ oracle on {used} "
                      f"host threads over token ranges, {dts:.1f} s",
            "cpu_model": cpu_model(),
            "single_thread": {"value": vec1 / 16 / dt1, "unit": UNIT, "cores": 1,
                              "sample": f"{vec1} vectors, one thread, {dt1:.1f} s"}}


def run_ours(args):
    dist = Dist(args.gpus)
    torch.cuda.set_device(dist.local)
    if args.only:
        fn = {"quantize": bench_quantize, "decode": bench_decode, "nsn": bench_nsn, "sweep": bench_sweep}[args.only]
        r = fn(args, dist)
        r.pop("sample_input", None)
        if dist.rank == 0:
            print(json.dumps({"only": args.only, **r}), flush=True)
        dist.close()
        return
    q = bench_quantize(args, dist)
    sweep = None if args.no_sweep else bench_sweep(args, dist)
    nsn = None if args.no_nsn else bench_nsn(args, dist)
    dec = None if args.no_decode else bench_decode(args, dist)
    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu:
        cpu = cpu_baseline(q["sample_input"], args.cpu_vectors)
    if dist.rank == 0:
        value = whole_job_rate(dist.world, q["tokens_per_step"] * args.steps, q["ms"])
        # The long per-configuration sweep goes first and the headline figures last, so that
        # a reader who keeps only the end of the line still has both halves of the metric.
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": dist.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": q["ms"] / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "llama3-8b-layer KV quantize: 8 KV heads x 32768 tokens x d128, bf16 K and V, "
                                   "2-bit Lloyd-Max + 1-bit QJL (m=128)",
                       "token": "one position of the layer = 8 heads x (K + V) = 16 vectors",
                       "layouts": "K one record per token, V bit planes in blocks of 32 tokens (what decode reads)",
                       "vectors_per_step": q["vectors_per_step"],
                       "l2": "4 rotating input copies per rank (4 x 134 MB > 126 MB L2)",
                       "parallelism": f"dp{dist.world} (independent layers per rank, no collective)"},
        }
        if sweep is not None:
            line["sweep"] = sweep
        if nsn is not None:
            line["nsn_quantize"] = nsn
        line["tensor"] = q["tensor"]
        line["rotation"] = q["rotation"]
        line["parity_boundary"] = parity_record()
        if dec is not None:
            line["decode_attn"] = dec
        line.update({"cpu_baseline": cpu, "e2e": q["e2e"], "gpu_launches": q["launches"], "clocks": q["clocks"],
                     "roofline": q["roofline"]})
        if dec is not None:
            line["decode_gbs"] = dec["value"]
            line["decode_frac_of_hbm"] = dec["frac_of_hbm"]
        print(json.dumps(line), flush=True)
    dist.close()


def run_reference(args):
    """The oracle on the host cores, same metric/unit/config, bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from calibration_free_rotated_token_b200 import workloads as wl

    c = wl.LLAMA_LAYER
    k = oracle.make_constants(c["d"], c["b"], c["handle_seed"])
    cores = os.cpu_count() or 1
    pos = 64 * cores                 # positions per step: 64 per host thread
    per_step = 16 * pos              # vectors per step: 8 heads of K and of V per position
    K = wl.llama_keys(c["heads"], pos, c["d"], c["k_seed"]).reshape(-1, c["d"]).double().numpy()
    V = wl.llama_values(c["heads"], pos, c["d"], c["v_seed"]).reshape(-1, c["d"]).double().numpy()
    for i in range(args.warmup):
        oracle_quantize_sharded(k, K, True, cores)
        oracle_quantize_sharded(k, V, True, cores)
    t0 = time.perf_counter()
    for i in range(args.steps):
        used = oracle_quantize_sharded(k, K, True, cores)
        oracle_quantize_sharded(k, V, True, cores)
    dt = time.perf_counter() - t0
    value = per_step / 16 * args.steps / dt
    sample = (f"{per_step} vectors ({pos} tokens) of the layer's K and V per step, fp64 C++ oracle on {used} host "
              f"threads over token ranges ({cpu_model()})")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": "llama3-8b-layer KV quantize: 8 KV heads x 32768 tokens x d128, bf16 K and V, "
                                   "2-bit Lloyd-Max + 1-bit QJL (m=128)",
                       "token": "one position of the layer = 8 heads x (K + V) = 16 vectors"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
