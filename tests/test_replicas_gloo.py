"""The N > 1 path of the benchmark: independent replicas whose timing is the
maximum over ranks and whose throughput is the sum over ranks (two gloo
ranks on CPU)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    ms = 10.0 + 5.0 * rank                   # rank 1 is the slow one
    m = bench.max_over_ranks(ms)
    v = bench.replica_throughput(world, 4, 100, m)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, m, v))


def test_two_replicas_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in out:
        assert m == 15.0
        assert v == pytest.approx(2 * 4 * 100 / 0.015)


def test_single_process_is_its_own_max():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
