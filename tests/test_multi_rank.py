"""The bench's multi-rank logic on CPU with the gloo backend, world size 2:
every rank runs its own replica (weak scaling), the step time is the max over
ranks, and the job throughput counts all ranks' work."""
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


def _rank(rank, world, port, out):
    import datetime
    import sys

    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    w, r, l = bench.dist_env()
    assert (w, r, l) == (world, rank, rank)
    bench.barrier()
    my_time = 0.010 + 0.005 * rank          # rank 1 is the slow one
    t = bench.reduce_max(my_time)
    v = bench.job_throughput(2.0e12, world, t)
    out.put((rank, t, v))
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_sum_the_work():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, t, v in res:
        assert t == pytest.approx(0.015)
        assert v == pytest.approx(2.0e12 * 2 / 0.015 / 1e12)


def test_single_process_needs_no_process_group():
    import bench
    assert bench.reduce_max(0.25) == 0.25
    assert bench.job_throughput(1e12, 1, 0.5) == pytest.approx(2.0)
