"""Host logic of the multi-rank bench on CPU: two `gloo` ranks on 127.0.0.1.

Each rank times its own batch (independent sequences, no data-path collective); the job
value uses the slowest rank's time, reduced with a MAX all-reduce that every rank calls in
the same order; only rank 0 prints.  These tests run that logic without a GPU.
"""
from __future__ import annotations

import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [10.0, 12.5][rank]               # rank 1 is the slow one
        ms = bench.reduce_max(local_ms, world, "cpu")
        dist.barrier()
        value, unit, hib = bench.job_value("csa", world, 8192, 20, ms)
        dec = bench.job_value("decode", world, 64, 20, ms)
        q.put((rank, ms, value, unit, hib, dec))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for rank, ms, value, unit, hib, dec in out:
        assert ms == 12.5                                   # max over ranks, seen by both
        assert unit == "tokens/s" and hib
        assert value == pytest.approx(2 * 8192 * 20 / 12.5e-3)  # both ranks' tokens / slowest time
        assert dec[1] == "us/step" and dec[0] == pytest.approx(12.5 / 20 * 1e3) and not dec[2]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.0, 1, "cpu") == 3.0
    assert bench.job_value("hca", 1, 100, 4, 2.0)[0] == pytest.approx(100 * 4 / 2e-3)


def test_reference_arm_prints_only_on_rank_zero(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    import synth

    class Args:
        warmup, steps, ref_budget, gpus = 0, 1, 0.01, 2

    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(Args, synth.WORKLOADS["tiny_csa_f32"])
    assert buf.getvalue() == ""
