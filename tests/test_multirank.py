"""The N > 1 host path of bench.py on CPU ranks (gloo, world size 2): replica batches differ
per rank, the barrier holds, and the step time is the maximum over ranks."""
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from workloads import WORKLOADS
    r, local, w = bench.dist_env()
    assert (r, local, w) == (rank, rank, world)
    bench.init_dist(w, "gloo")
    bench.barrier(w)
    t_max = bench.max_over_ranks(1.0 + rank, w, "cpu")
    total = bench.sum_over_ranks(float(rank + 1), w, "cpu")
    wl = WORKLOADS["tiny"]
    x = bench.rank_batch(wl, 1)
    out[rank] = (t_max, total, float(x.float().sum()))
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()   # no fork of this (multi-threaded) process
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 2.0          # slowest rank's time
    assert out[0][1] == out[1][1] == 3.0
    assert out[0][2] == out[1][2]                 # the same seeded batch on every process
    import bench
    from workloads import WORKLOADS, make_inputs
    wl = WORKLOADS["tiny"]
    x0 = make_inputs(wl).x
    assert not torch.equal(bench.rank_batch(wl, 1), x0)   # replicas see different tokens
