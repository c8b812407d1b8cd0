"""Multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2).

Covers what the N-GPU bench run relies on: the max-over-ranks reduction of
device times, distinct per-rank cache shards (weak scaling, no collective on
the data path), and that only rank 0 runs and prints the reference arm.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        r, wsize, local = bench.dist_env()
        t = bench.max_over_ranks(10.0 + 5.0 * rank, wsize)
        bench.barrier(wsize)
        seed = bench.shard_seed_offset(r)
        ref = bench.run_reference(bench.parse(["--impl", "reference", "--steps", "1",
                                               "--warmup", "0", "--ref-step-seconds", "0.05"]))
        q.put((r, wsize, t, seed, ref is not None))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    got = sorted(q.get() for _ in range(world))
    assert [g[0] for g in got] == [0, 1]
    assert all(g[1] == 2 for g in got)
    assert all(g[2] == 15.0 for g in got), "max over ranks"
    assert got[0][3] != got[1][3], "ranks must draw different shards"
    assert got[0][4] is True and got[1][4] is False, "reference arm runs on rank 0 only"
