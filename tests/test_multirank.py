"""The multi-GPU bench path on the CPU: world-size-2 gloo ranks.

bench.py runs one independent replica per rank (the attention path needs no
collective); the only cross-rank steps are the barrier and the max-over-ranks
reduction of the timed region.  These tests run those steps with the gloo
backend and check the whole-job throughput arithmetic.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, times, q):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    t = bench.max_over_ranks(times[rank], world)
    value = bench.aggregate(100.0, world, t)
    bench.barrier(world)
    dist.destroy_process_group()
    q.put((rank, t, value))


@pytest.mark.parametrize("times", [(2.0, 3.0), (5.0, 1.0)])
def test_two_rank_max_and_aggregate(times):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, value in out:
        assert t == max(times)
        assert value == pytest.approx(100.0 * 2 / max(times))


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.5, 1) == 1.5
    assert bench.aggregate(10.0, 1, 2.0) == 5.0
