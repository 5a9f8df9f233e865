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


def _fake_timer(wl, args, rank, world, device, cpu_seconds, cpu_tokens):
    """One rank's raw timings without a GPU: rank r's steps take (r + 1) ms, so the
    reduction over ranks must report the slower rank."""
    import bench
    import numpy as np
    bench.barrier(world)
    counts = np.bincount(np.arange(wl.T * wl.k) % wl.E, minlength=wl.E)   # balanced load
    return {"step_ms": [1.0 + rank] * args.steps, "stage_ms": [0.1 * (rank + 1)] * 6,
            "e2e_ms": [2.0 + rank] * args.steps, "counts": counts,
            "clocks": {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0},
            "kernels_per_step": 8, "h2d_bytes": wl.T * wl.d * 2, "d2h_bytes": wl.T * wl.d * 2,
            "fp8": wl.weights == "fp8"}


def _bench_worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    args = bench.parse_args(["--gpus", str(world), "--steps", "4", "--warmup", "3",
                             "--workloads", "prefill,decode_fp8"])
    r, local, w = bench.dist_env()
    bench.init_dist(w, "gloo")
    line = bench.run_ours(args, r, local, w, device="cpu", timer=_fake_timer,
                          stage_names=("router", "dispatch", "gather", "gate_up_gemm",
                                       "down_gemm", "combine"))
    out[rank] = line
    torch.distributed.destroy_process_group()


def test_bench_line_of_two_gloo_ranks():
    """bench.py's rank-level path on two CPU ranks (the GPU timing replaced by a fixed one):
    every rank reduces the same numbers, n_gpus is 2, the step time is the slower rank's,
    tokens count both ranks, and every extra workload gets its own entry."""
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_bench_worker, args=(world, port, out), nprocs=world, join=True)
    line = out[0]
    assert out[1]["value"] == line["value"]
    assert line["n_gpus"] == 2 and line["scaling"] == "weak"
    assert line["ms_per_step"] == 2.0                     # rank 1's (slower) steps
    assert line["value"] == 16 * 2 / 2.0e-3               # decode tokens of both ranks / time
    assert line["e2e"]["value"] == round(16 * 2 / 3.0e-3, 1)
    assert line["config"]["parallelism"] == "replicas2"
    assert sorted(line["workloads"]) == ["decode_fp8", "prefill"]
    pre = line["workloads"]["prefill"]
    assert pre["ms_per_step"] == 2.0 and pre["value"] == 8192 * 2 / 2.0e-3
    assert pre["roofline"]["bound"] == "tensor" and "frac_sustained" in pre["roofline"]
    assert line["workloads"]["decode_fp8"]["roofline"]["bound"] == "hbm"
    assert "cpu_baseline" not in line                     # only on a one-GPU run


def test_gpus_n_starts_n_ranks_through_torchrun_or_fails_loudly():
    import subprocess
    import sys
    import bench
    cmd = bench.launch_command(4, ["--gpus", "4", "--steps", "5"], 29511)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "5"] and cmd[-5].endswith("bench.py")
    # without enough visible GPUs the script stops before starting anything
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    env.pop("WORLD_SIZE", None)
    r = subprocess.run([sys.executable, bench.__file__, "--gpus", "2"], capture_output=True,
                       text=True, env=env, timeout=300)
    assert r.returncode != 0 and "--gpus 2 asked for" in r.stderr


def _shard_worker(rank: int, world: int, port: int, parallel: str, out):
    """One rank of a sharded layer on the CPU: its shard of the tiny workload through the
    oracle, the parts exchanged with the collective bench.py uses, added in rank order."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import numpy as np
    import bench
    import oracle
    from workloads import WORKLOADS, make_inputs
    bench.init_dist(world, "gloo")
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl)
    plan = bench.shard_plan(parallel, rank, world, wl.E, wl.F)
    (Wg, Wu, Wd), (Sg, Su, Sd) = bench.shard_weights(inp, plan)
    logits = oracle.router_logits(inp.x, inp.W_router, inp.bias)
    idx, w, _ = oracle.route(logits, wl.k)
    part = oracle.shard_output(inp.x, idx, w, Wg, Wu, Wd, Sg, Su, Sd, expert_begin=plan["e0"])
    parts = bench.gather_parts(torch.from_numpy(part), world)
    total = np.zeros_like(part)
    for p in parts:                      # rank order, as moe_reduce_partials adds them
        total += p.numpy()
    out[rank] = (plan, total)
    torch.distributed.destroy_process_group()


def test_sharded_layer_on_two_gloo_ranks():
    """tp and ep shard plans over two ranks: the shards cover the layer exactly once, and the
    all-gathered parts add up on every rank to the oracle's whole layer."""
    import numpy as np
    import oracle
    from workloads import WORKLOADS, make_inputs
    wl = WORKLOADS["tiny"]
    full = oracle.forward(make_inputs(wl))["y"]
    for parallel in ("tp", "ep"):
        world, port = 2, _free_port()
        mgr = mp.get_context("spawn").Manager()
        out = mgr.dict()
        mp.spawn(_shard_worker, args=(world, port, parallel, out), nprocs=world, join=True)
        plans = [out[r][0] for r in range(world)]
        if parallel == "tp":
            assert [(p["f0"], p["f1"]) for p in plans] == [(0, 64), (64, 128)]
            assert all(p["shared"] and p["n"] == wl.E for p in plans)
        else:
            assert [(p["e0"], p["n"]) for p in plans] == [(0, 8), (8, 8)]
            assert [p["shared"] for p in plans] == [True, False]
        for r in range(world):
            np.testing.assert_allclose(out[r][1], full, rtol=1e-11, atol=1e-12)


def test_shard_plans_cover_the_hy4_layer():
    import bench
    for world in (1, 2, 4, 8):
        tp = [bench.shard_plan("tp", r, world, 256, 2048) for r in range(world)]
        assert tp[0]["f0"] == 0 and tp[-1]["f1"] == 2048
        assert all(a["f1"] == b["f0"] for a, b in zip(tp, tp[1:]))
        ep = [bench.shard_plan("ep", r, world, 256, 2048) for r in range(world)]
        assert sum(p["n"] for p in ep) == 256 and sum(p["shared"] for p in ep) == 1
    import pytest
    with pytest.raises(ValueError):
        bench.shard_plan("tp", 0, 3, 256, 2048)     # 2048 / 3 is not a multiple of 64
