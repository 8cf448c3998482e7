"""The multi-GPU benchmark path on CPU: two gloo ranks (no GPU).

Attention heads are independent, so N ranks each own a disjoint slab of heads
and run the whole path on it with no data-path collective; the only collective
is the max over ranks of the device time.  These tests cover that host logic.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    try:
        r, w, d = bench.dist_setup(world)
        assert (r, w) == (rank, world) and d is not None
        w_ = W.get("tiny")
        heads = bench.head_shard(w_.H, r)
        # every rank draws its own heads; the two shards are disjoint and contiguous
        got = [None] * world
        dist.all_gather_object(got, list(heads))
        flat = sum(got, [])
        assert flat == list(range(world * w_.H))
        q, k, v = W.make_qkv(w_, 0, heads=heads)
        m = W.make_mask(w_, 0, heads=heads)
        # the shard equals the same heads of a single (world*H)-head job
        big = w_.with_(H=world * w_.H)
        qa, _, _ = W.make_qkv(big, 0, heads=heads)
        assert torch.equal(q, qa)
        assert np.array_equal(m, W.make_mask(big, 0, heads=heads))
        # slowest rank decides the time; throughput counts all ranks' work
        my_ms = 10.0 + 5.0 * rank
        mx = bench.reduce_max(my_ms, d)
        assert mx == 10.0 + 5.0 * (world - 1)
        bench.barrier(d)
        val = bench.job_throughput(w, 1e12, mx)
        assert abs(val - w * 1e12 / (mx * 1e-3) / 1e12) < 1e-9
        dist.destroy_process_group()
        results.put((rank, "ok"))
    except Exception as e:  # pragma: no cover - reported to the parent
        results.put((rank, repr(e)))


@pytest.mark.parametrize("world", [2])
def test_two_gloo_ranks_shard_heads(world):
    ctx = mp.get_context("spawn")
    results_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results_q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [results_q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    assert sorted(results) == [(r, "ok") for r in range(world)], results


def test_single_rank_needs_no_process_group():
    assert bench.dist_setup(1) == (0, 1, None)
    assert bench.reduce_max(3.5, None) == 3.5
    assert list(bench.head_shard(40, 0)) == list(range(40))
    assert list(bench.head_shard(40, 3)) == list(range(120, 160))
