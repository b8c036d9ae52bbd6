"""The benchmark's multi-rank path on the CPU: two gloo ranks on 127.0.0.1.

bench.py --gpus N runs one replica of the workload per rank (the path has
no exchange step), takes the slowest rank's device time and reports the
whole job's throughput; under torchrun the reference arm runs on rank 0
only.  These tests drive those host-side pieces with world size 2 and no
GPU: the max-over-ranks reduction, the whole-job value, the per-rank seeds,
and the reference arm's rank split (rank 0 prints one JSON line, rank 1
nothing)."""
import contextlib
import io
import json
import os
import socket
import types

import torch.multiprocessing as mp

import bench
from exact_io_aware_92_b200 import workloads as wl


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, wsize, local = bench.dist_env()
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms_max = bench.reduce_max(local_ms, "cpu")
        value = bench.job_throughput(1e12, 4, ms_max, wsize)
        seed = bench.replica_seed(wl.TINY, r)
        args = types.SimpleNamespace(warmup=0, steps=1, ref_budget=0.05)
        out = io.StringIO()
        with contextlib.redirect_stdout(out):
            rc = bench.run_reference(args, wl.TINY)
        dist.barrier()
        queue.put((r, wsize, local, ms_max, value, seed, rc, out.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    seeds = set()
    for r, wsize, local, ms_max, value, seed, rc, out in results:
        assert (wsize, local) == (2, r)
        assert ms_max == 15.0                      # the slowest rank's time, on both ranks
        assert abs(value - 2 * 1e12 * 4 / 15e-3 / 1e12) < 1e-9
        assert rc == 0
        seeds.add(seed)
        if r == 0:
            line = json.loads(out.strip())
            assert line["impl"] == "reference" and line["n_gpus"] == 2
            assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
        else:
            assert out == ""                        # other ranks exit without work
    assert len(seeds) == 2                          # each rank draws its own replica


def test_single_process_needs_no_group():
    assert bench.reduce_max(3.5, "cpu") == 3.5
    assert bench.job_throughput(2e12, 10, 1000.0, 1) == 20.0


def _shard_worker(rank, world, port, queue):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, Hq, Hkv, N, d = 2, 8, 4, 5, 3
        full = torch.arange(B * Hq * N * d, dtype=torch.float32).reshape(B, Hq, N, d)
        g0, g1, h0, h1 = bench.head_shard(Hkv, Hq // Hkv, world, rank)
        mine = full[:, h0:h1].contiguous()  # what this rank computes
        parts = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(parts, mine)
        queue.put((rank, (g0, g1, h0, h1), bool(torch.equal(bench.assemble_heads(parts), full))))
    finally:
        dist.destroy_process_group()


def test_head_shards_cover_the_problem_and_gather_back():
    """--shard heads: the ranks' kv-head blocks tile [0, Hkv), each with the
    query heads that share it, and the all-gathered slices reassemble O."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in results] == [(0, 2, 0, 4), (2, 4, 4, 8)]
    assert all(r[2] for r in results)


def test_head_shard_rejects_uneven_splits():
    import pytest
    with pytest.raises(ValueError):
        bench.head_shard(8, 4, 3, 0)
    assert bench.head_shard(8, 4, 8, 7) == (7, 8, 28, 32)
