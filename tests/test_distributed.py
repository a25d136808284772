"""Multi-rank bookkeeping of bench.py on CPU (gloo, world size 2).

The hot path has no exchange step: every rank runs an independent replica of
the workload (weak scaling) and only the timing is combined, as the maximum
over ranks.  These tests run two gloo ranks on the host.
"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # each rank times a different duration; the job time is the slowest one
        mx = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        value = bench.aggregate_value(1000, 4, mx, world)
        # the reference arm prints its line on rank 0 only
        args = type("A", (), {"workload": "16k", "steps": 2, "warmup": 1, "gpus": world})()
        buf = io.StringIO()
        with redirect_stdout(buf):
            bench.run_reference(args, world, rank)
        q.put((rank, mx, value, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_combine_timing_and_print_once():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, mx, value, out in res:
        assert mx == 15.0                                   # max over ranks
        assert value == pytest.approx(2 * 1000 * 4 / 15e-3)
    assert res[1][3] == ""                                  # rank 1 prints nothing
    line = json.loads(res[0][3].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
