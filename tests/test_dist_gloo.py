"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

bench.py --gpus N runs one process per GPU, each decoding its own seeded
batch (weak scaling, no collective on the data path); only the timing
reduction (max of the per-rank time, sum of the tokens) and the barriers
cross ranks.  Those are exercised here with the gloo backend.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        dev = torch.device("cpu")
        bench.barrier(dev)
        mx = bench.reduce_max(10.0 + rank * 5.0, dev)
        sm = bench.reduce_sum(8.0, dev)
        seeds = bench.rank_seed(1003, rank)
        env = bench.dist_env()
        q.put((rank, mx, sm, seeds, env))
    finally:
        dist.destroy_process_group()


def test_bench_rank_reductions_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, mx, sm, seed, env in res:
        assert mx == 15.0          # max over ranks of the per-rank time
        assert sm == 16.0          # total tokens of both ranks
        assert env == (rank, world, 0)
    assert res[0][3] != res[1][3]  # every rank decodes its own batch


def test_single_process_reductions_are_identity():
    import bench
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5
    assert bench.reduce_sum(2.0, torch.device("cpu")) == 2.0
