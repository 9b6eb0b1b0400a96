"""The N > 1 path of the bench on CPU: two gloo ranks exercise the weak-scaling helpers
(distinct per-rank batches, device time = max over ranks, whole-job aggregation)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    import datetime
    import bench
    from partial_activation_sync_caat_b200 import inputs as I
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.rank_env()
        assert (w, r, lr) == (world, rank, rank)
        # each rank draws its own batch (independent problems)
        d = I.make_rowpar_inputs(4, 32, 16, 2, seed=bench.rank_seed(rank))
        gathered = [torch.zeros_like(d["X"]) for _ in range(world)]
        dist.all_gather(gathered, d["X"])
        distinct = not torch.equal(gathered[0], gathered[1])
        # device time of the job = slowest rank
        my_ms = 1.0 + rank * 0.5
        mx = bench.max_over_ranks(my_ms, device="cpu")
        value = bench.whole_job_tflops(1e9, world, mx)
        out[rank] = (distinct, mx, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling_helpers():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()  # no fork of this (threaded) process
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
    for rank in range(world):
        distinct, mx, value = out[rank]
        assert distinct
        assert mx == pytest.approx(1.5)
        assert value == pytest.approx(2 * 1e9 / 1.5 / 1e9)


def test_single_process_defaults():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, device="cpu") == 3.25
    assert bench.whole_job_tflops(2e12, 1, 1.0) == pytest.approx(2000.0)
