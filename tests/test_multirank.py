"""Host logic of the multi-GPU benchmark path, on CPU with two gloo ranks.

The decode step has no exchange between sequences, so N GPUs run N replicas on
disjoint sequences and the only collective is the max-over-ranks timing
reduction; these tests run that reduction and the rank-0-only reporting."""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        m = bench.reduce_max_ms(ms, world, torch.device("cpu"))
        q.put((rank, m, bench.aggregate_value(world, 64, 20, m)))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_timing_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]  # both ranks report the slowest rank's time
    assert res[0][2] == pytest.approx(2 * 64 * 20 / 15e-3)


def test_single_rank_needs_no_process_group():
    import torch

    import bench
    assert bench.reduce_max_ms(7.5, 1, torch.device("cpu")) == 7.5
    assert bench.aggregate_value(1, 8, 10, 2.0) == pytest.approx(40000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import bench

    called = []
    monkeypatch.setattr(bench, "oracle_sample", lambda *a, **k: called.append(1) or (1.0, 1, "x"))

    class Args:
        host_groups, seed, warmup, steps, gpus, workload = 2, 0, 1, 1, 2, "offload28-128k"

    bench.run_reference(Args, dict(bench.WORKLOADS["offload28-128k"]), rank=1)
    assert called == []
