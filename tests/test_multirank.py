"""Host logic of the N > 1 bench path on CPU: world-size-2 gloo ranks (no GPU).

Every rank times its own replica; the job's time is the slowest rank's, and
the whole-job throughput counts every rank's tokens."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from nvfp4_mixture_experts_grouped_b200 import inputs


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        my_ms = 1.5 + rank  # rank 1 is the slow one
        ms = bench.max_over_ranks(torch, dist, my_ms, "cpu")
        q.put((rank, ms, bench.job_tokens_per_s(8192, world, ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, tps in res:
        assert ms == pytest.approx(2.5)  # the slowest rank's time on every rank
        assert tps == pytest.approx(2 * 8192 / 2.5e-3)


def test_single_process_keeps_own_time():
    assert bench.max_over_ranks(torch, None, 3.25, "cpu") == 3.25
    assert bench.job_tokens_per_s(16, 1, 2.0) == pytest.approx(8000.0)


def test_rank_batches_differ_weights_shared():
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.moe_inputs(wl)
    x0, l0 = bench.rank_batch(wl, d, 0)
    x1, l1 = bench.rank_batch(wl, d, 1)
    x1b, l1b = bench.rank_batch(wl, d, 1)
    assert x0 is d["x"] and l0 is d["logits"]
    assert x1.shape == x0.shape and l1.shape == l0.shape
    assert not np.array_equal(x0, x1) and not np.array_equal(l0, l1)
    assert np.array_equal(x1, x1b) and np.array_equal(l1, l1b)  # seeded per rank


def test_reference_arm_other_ranks_do_no_work(capsys):
    class A:
        tokens = experts = 0
        workload = "prefill"
        warmup = steps = 1
        cpu_sample_tokens = 1

    bench.run_reference(A(), rank=1, world=2)
    assert capsys.readouterr().out == ""
