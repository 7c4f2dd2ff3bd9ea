"""The multi-GPU path is replicas only (token-choice routing and the expert
FFNs are per token; every rank runs its own batch, no data-path collective).
What the benchmark does across ranks -- the max over ranks of the step time
and the whole-job throughput -- is checked here with two gloo ranks on CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [2.0, 3.5][rank]  # rank 1 is the slow replica
        ms = bench.max_over_ranks(local_ms, world, device="cpu")
        out[rank] = (ms, bench.replica_throughput(1000, world, ms))
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank_and_the_sum_of_tokens():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    for r in range(world):
        ms, tps = res[r]
        assert ms == 3.5
        assert tps == pytest.approx(2 * 1000 / 3.5e-3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(1.25, 1) == 1.25
    assert bench.replica_throughput(2048, 1, 2.0) == pytest.approx(1.024e6)
