"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo.

Each GPU rank of the benchmark runs its own replica; the only collectives are
the barrier around the timed region and the max over ranks of the elapsed
times.  Here two CPU processes exercise exactly those helpers."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import torch.distributed as dist

    class A:
        gpus = world
    w, r, l = bench.dist_setup(A())
    assert (w, r, l) == (world, rank, rank)
    bench.barrier(w)
    got = bench.reduce_max(1.5 + rank * 2.0, w, "cpu")
    bench.barrier(w)
    dist.destroy_process_group()
    q.put((rank, got))


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 3.5, 1: 3.5}


def test_reference_arm_non_zero_ranks_exit_without_work():
    import bench

    class A:
        steps, warmup, gpus = 1, 3, 2
    assert bench.run_reference(A(), 2, 1) == 0
