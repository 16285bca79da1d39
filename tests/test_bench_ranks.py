"""bench.py's multi-process timing on CPU: two gloo ranks agree on the slowest rank's
time and on the whole-job throughput (the path torchrun takes for --gpus N > 1)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([10.0 + rank, 5.0 - rank, 1.0 * rank])
        out[rank] = (got, bench.whole_job_tflops(4e12, world, got[0]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:     # no fork of this multi-threaded process
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        got, tflops = res[rank]
        assert got == [11.0, 5.0, 1.0]
        assert tflops == pytest.approx(2 * 4e12 / 11e-3 / 1e12)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 1.5]) == [3.0, 1.5]
    assert bench.whole_job_tflops(2e12, 1, 2.0) == pytest.approx(1000.0)
