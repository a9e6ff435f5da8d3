"""Multi-process (world size 2, gloo, CPU) checks of the bench's replica logic:
the step time is the slowest rank's, the whole-job weight-stream rate counts
every replica's own weight pass, and no data-path collective is involved."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        my_ms = [3.0, 5.5][rank]
        slowest = bench.max_over_ranks(my_ms, world)
        bench.barrier(world)
        out[rank] = (slowest, bench.weight_stream_gbs(10 ** 9, world, slowest))
    finally:
        dist.destroy_process_group()


def test_replica_timing_and_aggregate_rate():
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, _free_port(), out), nprocs=2, join=True)
    for r in (0, 1):
        slowest, gbs = out[r]
        assert slowest == 5.5
        assert gbs == pytest.approx(2 * 1e9 / 5.5e-3 / 1e9)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(7.0, 1) == 7.0
    assert bench.weight_stream_gbs(13_741_588_480, 1, 2.0) == pytest.approx(6870.79424)
