"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the
whole-job throughput is every rank's tokens over the slowest rank's time, and
every rank sees the same reduced numbers."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    bench.init_dist(world, "gloo")
    w, r, l = bench.dist_env()
    units = 32.0 * (rank + 1)           # rank 0: 32 tokens, rank 1: 64 tokens
    secs = 0.5 + rank                   # rank 1 is the slower one
    value, slowest = bench.job_throughput(units, secs, world)
    bench.barrier(world)
    q.put((rank, w, r, value, slowest))
    dist.destroy_process_group()


def test_job_throughput_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, world, r, value, slowest in got:
        assert world == 2 and r == rank
        assert slowest == 1.5
        assert abs(value - (32.0 + 64.0) / 1.5) < 1e-9


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_throughput(100.0, 2.0, 1) == (50.0, 2.0)
