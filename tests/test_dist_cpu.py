"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the max over
ranks of the per-rank elapsed times, the whole-job throughput built from it,
and the reference arm's rule that only rank 0 does work."""
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


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as td
    sys.path.insert(0, ROOT)
    import bench
    td.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                          timeout=datetime.timedelta(seconds=60))
    try:
        mine = [10.0 + 5.0 * rank, 3.0 - rank]  # rank 1 is the slow one for the first value
        got = bench.reduce_max_over_ranks(mine)
        val = bench.job_throughput(world, 354.0, 20, got[0])

        class A:
            steps, warmup, workload = 1, 0, "c1_1s_b1_d768"
        rc = bench.run_reference(A, rank, world) if rank != 0 else 0
        out[rank] = (got, val, rc)
    finally:
        td.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        got, val, rc = out[r]
        assert got == [15.0, 3.0]
        assert val == pytest.approx(2 * 354.0 * 20 / 0.015)
        assert rc == 0
