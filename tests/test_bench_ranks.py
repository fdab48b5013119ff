"""Multi-rank bench logic on CPU: two gloo ranks, as torchrun would start them (one process per
GPU, replicas only).  The job's step time must be the max over ranks and its throughput count
every rank's tokens."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, ms_by_rank, out):
    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_max, value = bench.replica_throughput(ms_by_rank[rank], 640, dist, device="cpu")
        out[rank] = (ms_max, value)
    finally:
        dist.destroy_process_group()


def test_replica_throughput_two_gloo_ranks():
    ctx = torch.multiprocessing.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    ms_by_rank = [12.5, 20.0]
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, ms_by_rank, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(2):
        ms_max, value = out[r]
        assert ms_max == 20.0
        assert value == pytest.approx(2 * 640 / 0.020)


def test_replica_throughput_single_process():
    import bench

    ms_max, value = bench.replica_throughput(8.0, 64, None)
    assert ms_max == 8.0 and value == pytest.approx(8000.0)
