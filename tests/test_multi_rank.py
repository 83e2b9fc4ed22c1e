"""Multi-process host logic of bench.py on CPU (gloo, world size 2): the whole-job
throughput is every rank's units over the slowest rank's time, and only rank 0
of the reference arm does any work."""
import argparse
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    bench.dist_init(world, "gloo")
    v, t = bench.aggregate(100.0, 1.0 + rank, world)
    bench.barrier(world)
    q.put((rank, v, t))
    dist.destroy_process_group()


def test_aggregate_is_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, v, t in got:
        assert t == 2.0            # the slower rank's time
        assert v == 100.0          # 2 ranks x 100 units / 2 s


def test_reference_arm_only_rank0_works(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.reference_arm(argparse.Namespace(steps=1, warmup=3, gpus=2))
    assert buf.getvalue() == ""
