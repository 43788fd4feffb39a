"""Host logic of the multi-process bench path on CPU: world size 2 over gloo.
Each rank reports its own device time; the job's time is the max over ranks,
and the barrier holds every rank until all arrive."""

import os
import socket

import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    ws, r, local = bench.dist_env()
    assert (ws, r, local) == (world, rank, rank)
    bench.init_dist(ws, "gloo")
    bench.barrier(ws)
    m = bench.max_over_ranks(10.0 + rank, ws, "cpu")
    out[rank] = m
    import torch.distributed as dist
    dist.destroy_process_group()


def test_max_over_ranks_world2():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    assert dict(out) == {0: 11.0, 1: 11.0}


def test_single_rank_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
