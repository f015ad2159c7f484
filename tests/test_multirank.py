"""Multi-rank host logic of the benchmark on CPU: two gloo ranks launched
the way torchrun does (RANK / WORLD_SIZE / MASTER_* in the environment).
The timed number is the max over ranks and the value counts every rank's
work; only rank 0 runs the reference arm."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench.dist_info()
        ms = 10.0 + 5.0 * rank             # rank 1 is the slow one
        m = bench.max_over_ranks(ms, torch.device("cpu"))
        v = bench.total_value_gbs(1_000_000_000, 4, ws, m)

        class A:
            steps, warmup = 1, 0
        import workloads
        tiny = workloads.WORKLOADS["tiny"]
        ref = bench.run_reference(A, tiny)
        q.put((rank, ws, r, local, m, v, ref is None))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q))
             for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ws, r, local, m, v, ref_none in res:
        assert ws == 2 and r == rank and local == rank
        assert m == 15.0                       # max over ranks
        assert abs(v - 2 * 4 * 1.0 / 0.015) < 1e-6   # GB/s of both ranks
        assert ref_none == (rank != 0)         # reference arm: rank 0 only
