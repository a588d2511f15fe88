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


# ---------------------------------------------------------------- head shards

def test_head_shards_cover_every_group_once():
    import exact_io_aware_44_b200 as fa
    for (B, Hq, Hkv) in ((2, 32, 32), (1, 32, 8), (3, 12, 4), (2, 8, 2)):
        for world in (1, 2, 3, 4, 8, 16):
            seen_q, seen_k = [], []
            for r in range(world):
                q0, q1, k0, k1 = fa.head_shard(B, Hq, Hkv, r, world)
                assert (q1 - q0) == (k1 - k0) * (Hq // Hkv)
                seen_q += list(range(q0, q1))
                seen_k += list(range(k0, k1))
            assert seen_q == list(range(B * Hq)) and seen_k == list(range(B * Hkv))
            sizes = [fa.head_shard(B, Hq, Hkv, r, world)[3] - fa.head_shard(B, Hq, Hkv, r, world)[2]
                     for r in range(world)]
            assert max(sizes) - min(sizes) <= 1


def _shard_rank(rank, world, port, out, kind="fwd"):
    """Each rank computes its head slice as an independent problem (B = 1) with
    the float64 oracle standing in for the kernel, then all ranks gather the
    slices: the result must equal the unsharded problem. kind "decode": a few
    new queries per head against a longer key/value cache."""
    import datetime
    import sys

    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import exact_io_aware_44_b200 as fa
    import oracle
    B, Hq, Hkv, N, d = 3, 8, 2, 19, 8
    Nq = 3 if kind == "decode" else N
    rng = np.random.default_rng(7)
    q, k, v = rng.standard_normal((B, Hq, Nq, d)), rng.standard_normal((B, Hkv, N, d)), rng.standard_normal((B, Hkv, N, d))
    fn = oracle.decode_fwd64 if kind == "decode" else oracle.attention_fwd64
    q0, q1, k0, k1 = fa.head_shard(B, Hq, Hkv, rank, world)
    qs = q.reshape(B * Hq, Nq, d)[q0:q1][None]
    ks = k.reshape(B * Hkv, N, d)[k0:k1][None]
    vs = v.reshape(B * Hkv, N, d)[k0:k1][None]
    o, lse = fn(qs, ks, vs, True, 0.3)
    parts = [None] * world
    dist.all_gather_object(parts, (q0, q1, o[0], lse[0]))
    full_o = np.concatenate([p[2] for p in sorted(parts, key=lambda p: p[0])]).reshape(B, Hq, Nq, d)
    full_l = np.concatenate([p[3] for p in sorted(parts, key=lambda p: p[0])]).reshape(B, Hq, Nq)
    ref_o, ref_l = fn(q, k, v, True, 0.3)
    out.put((rank, float(np.abs(full_o - ref_o).max()), float(np.abs(full_l - ref_l).max())))
    dist.destroy_process_group()


@pytest.mark.parametrize("kind", ["fwd", "decode"])
def test_two_gloo_ranks_head_sharded_problem_equals_the_whole(kind):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_rank, args=(r, world, port, q, kind)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for _ in range(world):
        rank, eo, el = q.get(timeout=10)
        assert eo < 1e-12 and el < 1e-12, (rank, eo, el)
