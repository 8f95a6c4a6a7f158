"""World-size-2 gloo checks of the benchmark's multi-process plumbing on CPU.

On several GPUs each rank runs an independent replica of the layer (the path shards into
independent problems; there is no collective on the data path).  What crosses ranks is the
timing: a barrier on both sides of the timed region and the max over ranks of each time.
"""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    dist = bench.init_dist(world, "gloo")
    bench.barrier(world)
    t = bench.reduce_max(1.5 + rank, world)
    u = bench.reduce_max(10.0 - rank, world)
    bench.barrier(world)
    out[rank] = (t, u)
    dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")  # no fork of this (multi-threaded) process anywhere
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == (2.5, 10.0) and out[1] == (2.5, 10.0)


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max(3.25, 1) == 3.25
    bench.barrier(1)
