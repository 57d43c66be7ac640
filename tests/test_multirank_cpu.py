"""The benchmark's N > 1 plumbing on CPU: two gloo ranks.

dgrad shards with no exchange step (every rank runs its own replica of the
workload), so the only cross-rank operations are the barrier around the timed
region and the max over ranks of the step time.  This runs both with
world_size 2 over gloo on 127.0.0.1 and checks the job-level aggregation.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    try:
        w, r, local = bench.dist_init()
        assert (w, r, local) == (world, rank, rank)
        bench.barrier(w)
        step_ms = 2.0 + rank          # rank 1 is the slow one
        mx = bench.max_over_ranks(w, step_ms)
        flops_per_rank = 1e9
        value = bench.job_throughput(flops_per_rank, w, mx)
        bench.barrier(w)
        q.put((rank, mx, value))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_job_total():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, mx, value in res:
        assert mx == 3.0                       # max over ranks
        assert abs(value - 2 * 1e9 / 3e-3 / 1e12) < 1e-9   # both ranks' work over the slowest time
