"""bench.py's replica plumbing with two ranks on the CPU (gloo backend).

N > 1 runs independent replicas that meet only around the timed region: each
rank's time is reduced with MAX and rank 0 reports.  This runs the same helpers
the GPU run uses (dist_setup, barrier, max_over_ranks, dist_teardown) in two
processes rendezvousing on 127.0.0.1.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    r, w, local, active = bench.dist_setup(world)
    try:
        bench.barrier(active)
        t = bench.max_over_ranks(1.5 + rank, active)       # rank r "took" 1.5 + r seconds
        out.put((r, w, local, active, t))
        bench.barrier(active)
    finally:
        bench.dist_teardown(active)


def test_two_ranks_report_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [x[0] for x in res] == [0, 1]
    for r, w, local, active, t in res:
        assert w == 2 and local == r and active
        assert t == 2.5                                        # max over ranks, on every rank


def test_single_process_needs_no_process_group(monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    sys.path.insert(0, ROOT)
    import bench
    assert bench.dist_setup(1) == (0, 1, 0, False)
    assert bench.max_over_ranks(3.0, False) == 3.0
