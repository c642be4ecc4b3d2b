"""Host logic of bench.py's multi-process (N > 1) path, run as two gloo ranks on the CPU.

The decode path shards as independent replicas (no data-path collective); what N > 1 adds is
the timing reduction (the slowest rank's time) and the rule that only rank 0 prints."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        slowest = bench.max_over_ranks(torch, dist, 1.5 + rank, device="cpu")
        out = io.StringIO()

        class A:
            steps, warmup, cpu_seconds, gpus = 1, 0, 0.0, world
        with redirect_stdout(out):
            if rank != 0:
                bench.run_reference(A, rank, world)   # other ranks exit without work
        q.put((rank, slowest, out.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_rank0_only():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        rank, slowest, printed = q.get(timeout=120)
        res[rank] = (slowest, printed)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == pytest.approx(2.5) and res[1][0] == pytest.approx(2.5)
    assert res[1][1] == ""


def test_end_to_end_split_covers_every_problem_once():
    sys.path.insert(0, ROOT)
    import bench
    for n in (0, 1, 3, 4, 7, 28, 252, 253):
        for parts in (1, 2, 4, 8):
            r = bench.split_ranges(n, parts)
            assert len(r) <= parts
            assert [i for a, b in r for i in range(a, b)] == list(range(n))
            assert all(b > a for a, b in r)
    assert bench.split_ranges(252, 4) == [(0, 63), (63, 126), (126, 189), (189, 252)]
