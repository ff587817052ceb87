"""The multi-rank plumbing of bench.py on CPU: two gloo ranks agree on the
maximum time, pass the barriers, and only rank 0 runs the reference arm."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench

    w, r, _ = bench.dist_setup("gloo")
    try:
        assert (w, r) == (world, rank)
        bench.barrier(w)
        got = bench.max_over_ranks(1.5 + rank, w, "cpu")
        bench.barrier(w)

        class A:
            workload, steps, warmup = 0, 1, 0

        ran = None
        if rank != 0:
            ran = bench.reference_arm(A, w, r)  # returns at once on ranks > 0
        q.put((rank, got, ran))
    finally:
        bench.dist_teardown(w)


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(100)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(world))
    assert [g for _, g, _ in res] == [2.5, 2.5]
    assert res[1][2] is None
