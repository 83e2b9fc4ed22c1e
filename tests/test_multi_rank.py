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


def test_reference_arm_line_contract(monkeypatch):
    # rank 0 of a one-process run: one JSON line with the contract's keys, the
    # oracle timed on this host's cores, no host<->device bytes
    import json
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.reference_arm(argparse.Namespace(steps=1, warmup=3, gpus=1))
    lines = [x for x in buf.getvalue().splitlines() if x.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] >= 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["config"]["workload"] == "decode_b16_ctx131072_14layers_cli2"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]
