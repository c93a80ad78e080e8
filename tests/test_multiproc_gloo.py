"""The replica bookkeeping of bench.py across 2 ranks on CPU (gloo): every
rank runs its own copy of the layer, the job's throughput is the work of all
ranks over the slowest rank's time, and no collective touches the data path."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    # rank r processed 1e12 * (r + 1) flops in 10 * (r + 1) ms
    tflops, max_ms, total = bench.aggregate(1e12 * (rank + 1), 10.0 * (rank + 1), world)
    out[rank] = (tflops, max_ms, total)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        tflops, max_ms, total = out[r]
        assert max_ms == 20.0
        assert total == 3e12
        assert tflops == pytest.approx(3e12 / 0.020 / 1e12)


def _worker_sharded(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    # a 6e12-flop batch split over the ranks; rank r took 10 + 5 r ms
    tflops, max_ms = bench.aggregate_sharded(6e12, 10.0 + 5.0 * rank, world)
    out[rank] = (tflops, max_ms)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_token_sharded_aggregation_gloo():
    """bench.py --sharded: the batch's work is counted once and divided by the
    slowest rank's time (strong scaling), on every rank alike."""
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker_sharded, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        tflops, max_ms = out[r]
        assert max_ms == 15.0
        assert tflops == pytest.approx(6e12 / 0.015 / 1e12)
