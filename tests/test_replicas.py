"""Several GPUs run independent replicas of the request (batch-1 decode has no split across
devices); the benchmark's only collective is the maximum of the measured times over ranks.
Checked here with two gloo ranks on the CPU."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        mine = [100.0 + 10.0 * rank, 5.0 - rank]  # per-rank times (ms)
        total, other = bench.max_over_ranks(mine, torch.device("cpu"))
        out.put((rank, total, other, bench.replica_throughput(1024, world, total)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_times_are_the_maximum_over_two_ranks_and_throughput_counts_every_replica():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, total, other, tput in got:
        assert total == 110.0 and other == 5.0  # element-wise max over ranks
        assert tput == pytest.approx(2 * 1024 / 0.110)


def test_single_rank_keeps_its_own_times():
    assert bench.max_over_ranks([3.5, 1.0], torch.device("cpu")) == [3.5, 1.0]
    assert bench.replica_throughput(1024, 1, 1000.0) == pytest.approx(1024.0)
