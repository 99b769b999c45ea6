"""The multi-process (N > 1) host path of bench.py on CPU: two gloo ranks.

bench.py runs one replica of the layer per GPU (weak scaling; the layer
shards by tokens, so no data-path collective exists).  What crosses ranks is
the timing protocol: a barrier and a synchronisation on both sides of the
timed region, the maximum of the device times over ranks, and the whole-job
value computed from it.  These tests run that protocol with gloo ranks on
the CPU, each rank reporting a different time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, local = bench.dist_env()
        calls = []
        ms = bench.timed_region(dist, lambda: 10.0 + 5.0 * r, lambda: calls.append("sync"))
        total = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        steps = 4
        value = bench.job_value(ws, 2.0e12, total / steps)
        out.put((r, ws, local, ms, total, value, calls))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_timing_protocol_max_over_ranks(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = 10.0 + 5.0 * (world - 1)
    for r, (rank, ws, local, ms, total, value, calls) in enumerate(res):
        assert (rank, ws, local) == (r, world, r)
        assert ms == 10.0 + 5.0 * r               # each rank's own time
        assert total == slowest                   # every rank reports the slowest rank's time
        # whole-job throughput: world replicas x 2e12 FLOP per step at slowest / 4 ms per step
        assert value == pytest.approx(world * 2.0e12 / (slowest / 4 * 1e-3) / 1e12)
        assert calls == ["sync", "sync"]          # synchronised on both sides


def test_single_rank_needs_no_process_group():
    assert bench.timed_region(None, lambda: 3.5, lambda: None) == 3.5
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5
    assert bench.job_value(1, 1.0e12, 1.0) == pytest.approx(1000.0)   # 1e12 FLOP per 1 ms step
