"""Multi-process plumbing of the benchmark (world size 2, gloo on CPU): max-over-ranks timing and weak scaling."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # each rank times its own replica; the job's time is the slowest rank's
        mine = [1.0 + rank, 10.0 - rank, 3.5]
        q.put((rank, bench.max_over_ranks(mine)))
    finally:
        dist.destroy_process_group()


def _shard_worker(rank, world, port, q):
    """What run_gpu does per rank, without the GPU: draw this rank's seeded inputs, time its replica (a fake
    duration that differs by rank), and aggregate with max_over_ranks into the weak-scaling value."""
    import hashlib

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from synth import mamba2_step_inputs
        wl = bench.rank_workload(rank).replace(batch=2)
        digest = hashlib.sha1(mamba2_step_inputs(wl, 0)["x"].tobytes()).hexdigest()
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        my_ms = 100.0 + 25.0 * rank
        total_ms = bench.max_over_ranks([my_ms])[0]
        value = bench.weak_scaling_value(bench.WL.batch, world, 64, total_ms)
        q.put((rank, digests, total_ms, value))
    finally:
        dist.destroy_process_group()


def test_rank_shards_and_weak_scaling_fields_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {r: rest for r, *rest in (q.get(timeout=120) for _ in procs)}
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    digests0, total0, value0 = out[0]
    digests1, total1, value1 = out[1]
    assert digests0 == digests1 and digests0[0] != digests0[1]     # each rank decodes its own shard
    assert total0 == total1 == 125.0                                # the slowest rank's time, on every rank
    assert value0 == value1 == pytest.approx(256 * 2 * 64 / 0.125)  # tokens of all ranks / that time


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0] == out[1] == [2.0, 10.0, 3.5]


def test_weak_scaling_value_and_single_process():
    import bench
    assert bench.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]          # not distributed: identity
    # 256 tokens per rank-step, 4 ranks, 100 steps in 50 ms on the slowest rank
    assert bench.weak_scaling_value(256, 4, 100, 50.0) == pytest.approx(256 * 4 * 100 / 0.05)
