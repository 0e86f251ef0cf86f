"""Host logic of the N > 1 bench path (independent replicas, no collective
on the data path) with two gloo ranks on the CPU: disjoint token streams,
max-over-ranks timing, whole-job throughput, rank-0-only reference arm."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        streams = bench.replica_streams(rank, 7)
        every = [None] * world
        dist.all_gather_object(every, streams)
        # each rank's own timing; the job takes the slowest
        mine = [10.0 + 5.0 * rank, 20.0 - 3.0 * rank]
        got = bench.max_over_ranks(mine, world, torch.device("cpu"))
        rate = bench.whole_job_rate(got[0], 100, world)
        out.put((rank, every, got, rate))
    finally:
        dist.destroy_process_group()


def test_two_replicas_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = {}
    for _ in range(world):
        r, every, got, rate = q.get(timeout=120)
        res[r] = (every, got, rate)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        every, got, rate = res[r]
        assert set(every[0]).isdisjoint(every[1])          # replicas decode different tokens
        assert len(set(every[0])) == 7 and len(set(every[1])) == 7
        assert got == [15.0, 20.0]                          # element-wise max over ranks
        assert rate == pytest.approx(100 * world / 0.015)   # all ranks' tokens / slowest time


def test_single_rank_needs_no_process_group():
    import torch
    assert bench.max_over_ranks([3.0, 4.0], 1, torch.device("cpu")) == [3.0, 4.0]
    assert bench.replica_streams(0, 3) == [1000, 1001, 1002]


def test_reference_arm_runs_on_rank0_only(capsys):
    class A:
        steps, warmup = 1, 3
    assert bench.run_reference(A(), 1, 2) is None
    assert capsys.readouterr().out == ""
