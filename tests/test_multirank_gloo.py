"""World-size-2 runs of the bench's multi-rank host logic on CPU (gloo).

The path partitions: every rank quantizes its own layer (decode: its own
sequences), so only a barrier and the max-over-ranks timing cross ranks.
These tests run that logic in two processes: the reduction returns the
slowest rank's time on every rank, the whole-job rate counts all ranks' work
over it, and the per-rank seeds give every rank different inputs.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from calibration_free_rotated_token_b200 import workloads as wl

    d = bench.Dist(world, backend="gloo")
    try:
        ms_here = 10.0 + 5.0 * rank          # rank 1 is the slow one
        d.barrier()
        ms = d.max(ms_here)
        c = wl.LLAMA_LAYER
        k = wl.llama_keys(1, 64, c["d"], c["k_seed"] + 1000 * d.rank)
        sl = wl.cache_slice_seed(c["handle_seed"], 0, d.rank, 0)
        out.put((rank, ms, bench.whole_job_rate(d.world, 1000.0, ms), float(k.double().sum()), sl))
    finally:
        d.close()


def test_two_ranks_agree_on_the_slowest_time_and_draw_different_inputs():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, rate0, k0, s0), (r1, ms1, rate1, k1, s1) = res
    assert ms0 == ms1 == 15.0                       # max over ranks, seen by every rank
    assert rate0 == rate1 == pytest.approx(2 * 1000.0 / 0.015)
    assert k0 != k1 and s0 != s1                    # independent work per rank


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    os.environ.pop("WORLD_SIZE", None)
    d = bench.Dist(1)
    assert d.pg is None and d.max(3.5) == 3.5
    d.barrier()
    assert bench.whole_job_rate(1, 500.0, 250.0) == 2000.0
