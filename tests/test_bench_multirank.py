"""The benchmark's multi-rank plumbing on CPU: two gloo ranks on 127.0.0.1.

Every rank runs its own copy of the workload (no data-path collective); the only
cross-rank steps are barriers and the max-over-ranks of the timed duration.
"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    try:
        w, r, _ = bench.dist_setup(None)
        assert (w, r) == (world, rank)
        # the slowest rank decides the time
        got = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        bench.barrier(world)
        # the reference arm prints from rank 0 only, other ranks do no work
        buf = io.StringIO()
        args = type("A", (), {"workload": "encoder", "steps": 1, "warmup": 0})()
        import workloads
        orig = bench.oracle_sample
        bench.oracle_sample = lambda *a, **k: (1.0, "stub sample", 1, 0.01)
        try:
            with redirect_stdout(buf):
                bench.run_reference(args, world, r)
        finally:
            bench.oracle_sample = orig
        q.put((rank, got, buf.getvalue()))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max_and_print_once():
    world, port = 2, free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=90) for _ in range(world)]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    results.sort()
    assert [r[1] for r in results] == [15.0, 15.0]
    out0, out1 = results[0][2], results[1][2]
    assert out1 == ""
    line = json.loads(out0.strip())
    assert line["impl"] == "reference" and line["n_gpus"] == world
    assert line["e2e"]["h2d_bytes_per_step"] == 0
