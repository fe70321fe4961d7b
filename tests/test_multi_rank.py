"""The N-GPU path of bench.py on CPU: two gloo ranks run the host logic that
shards the workload (one independent problem per rank, distinct seeds) and
times the job as the slowest rank (max over ranks)."""
import multiprocessing as mp
import os
import socket

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    from ss_inputs import fwd_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}",
                            timeout=datetime.timedelta(seconds=60))
    try:
        seed = bench.shard_seed(3, rank)
        inp = fwd_inputs(1, 8, 16, 16, "bf16", seed, "cpu")
        ms = 10.0 + 5.0 * rank
        dist.barrier()
        ms_max = bench.reduce_max(dist, ms, torch.device("cpu"))
        value = bench.aggregate_value(world, 1_000_000_000, 10, ms_max)
        q.put((rank, seed, float(inp["u"].float().sum()), ms_max, value))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_take_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    (r0, s0, u0, m0, v0), (r1, s1, u1, m1, v1) = out
    assert s0 != s1 and u0 != u1            # each rank draws its own problem
    assert m0 == m1 == 15.0                 # both see the slowest rank's time
    assert v0 == v1 == pytest.approx(2 * 1e9 * 10 / 15e-3 / 1e9)


def test_single_rank_helpers():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(None, 3.5, None) == 3.5
    assert bench.shard_seed(5, 0) == 5
    assert bench.aggregate_value(1, 2e9, 1, 1000.0) == pytest.approx(2.0)
