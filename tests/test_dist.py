"""The benchmark's multi-rank logic on CPU with gloo, world size 2: ranks agree
on the slowest rank's time and the whole-job value counts every rank's units
(weak scaling: each rank runs the same per-rank step on its own GPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 2.0 + rank            # rank 1 is slower
        slowest = bench.reduce_max(ms, world, torch.device("cpu"))
        value = bench.whole_job_value(1e9, world, slowest, "GB/s")
        out[rank] = (slowest, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_whole_job_value():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    slowest, value = res[0]
    assert slowest == 3.0
    # 2 ranks x 1e9 bytes in 3 ms = 666.67 GB/s
    assert value == pytest.approx(2e9 / 3e-3 / 1e9)


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max(1.25, 1, None) == 1.25
    assert bench.whole_job_value(6e9, 1, 2.0, "GB/s") == pytest.approx(3000.0)
    assert bench.whole_job_value(2e12, 1, 1.0, "TFLOP/s") == pytest.approx(2000.0)
