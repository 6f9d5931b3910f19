"""The multi-rank path of bench.py on CPU (gloo, world size 2): the layer has no exchange
between ranks (replicas), so the only cross-rank step is the timing reduction. Checked: every
rank ends with the maximum over ranks, the whole-job rate uses that maximum, and the
reference arm prints only on rank 0."""
import datetime
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import bench
        # Rank-dependent timings: rank 0 is slower on the first, rank 1 on the second.
        got = bench.max_over_ranks([10.0 - rank, 3.0 + 2 * rank], torch.device("cpu"), world)
        rate = bench.job_rate(world, 100, got[0])
        buf = io.StringIO()
        with redirect_stdout(buf):
            bench.run_reference(type("A", (), {"steps": 1, "warmup": 0})(), rank, world) if rank != 0 else None
        results.put((rank, got, rate, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_timing_reduction_over_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        rank, got, rate, printed = results.get(timeout=120)
        out[rank] = (got, rate, printed)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        got, rate, printed = out[rank]
        assert got == [10.0, 5.0]                       # max over ranks, elementwise
        assert rate == pytest.approx(2 * 100 / 0.010)   # all ranks' frames over the slowest time
    assert out[1][2] == ""                              # the reference arm is silent off rank 0


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5], torch.device("cpu"), 1) == [1.5, 2.5]
    assert bench.job_rate(1, 50, 1000.0) == pytest.approx(50.0)
