"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the slowest
rank's time is the job's time, the whole-job rate counts every rank's units,
and every rank draws its own batch of the same recipe."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    local = [10.0 + 5.0 * rank, 3.0 - rank]
    mx = bench.max_over_ranks(local)
    b = bench.make_workload("tiny", rank)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, mx, int(b.T), b.q[:4].tolist(), b.lengths.tolist()))


def test_two_rank_max_and_rates():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, mx0, T0, q0, L0), (r1, mx1, T1, q1, L1) = res
    assert mx0 == mx1 == [15.0, 3.0]
    assert q0 != q1 or L0 != L1                       # independent batches per rank
    import bench
    # 2 ranks x 10 steps x 100 units in 50 ms (slowest rank) = 40000 units/s
    assert bench.weak_scaling_rate(2, 10, 100, 50.0) == pytest.approx(40000.0)
