"""The multi-process plumbing of bench.py on CPU: world size 2 over gloo.

The sharded MLP runs as independent replicas (no data-path collective), so
the only cross-rank step is the timing reduction: every rank must receive the
maximum over ranks, and the whole-job throughput is world x per-step FLOPs /
slowest time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks([1.0 + rank, 10.0 - 3 * rank], dist, "cpu")
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_timing_is_max_over_ranks_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [2.0, 10.0]


def test_replica_throughput_is_weak_scaling():
    import bench
    one = bench.replica_throughput(1, 1.443e12, 1.0)
    assert one == pytest.approx(1443.0)
    assert bench.replica_throughput(8, 1.443e12, 1.0) == pytest.approx(8 * one)
    assert bench.replica_throughput(2, 1.443e12, 2.0) == pytest.approx(one)
