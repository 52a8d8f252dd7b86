"""CPU (gloo, world size 2) tests of the bench's multi-rank host logic: max-over-ranks
timing and whole-job throughput aggregation.  No GPU and no attention kernels are used."""

import os
import socket

import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.dist_env() == (rank, world, rank)
        t = 1.0 + rank  # rank 1 is slower
        t_max = bench.max_over_ranks(t, world)
        value = bench.throughput_tflops(2e12, steps=5, world=world, max_seconds=t_max)
        out[rank] = (t_max, value)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_throughput():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()   # no fork of this (multi-threaded) process
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    for rank in range(2):
        t_max, value = out[rank]
        assert t_max == 2.0                       # the slowest rank's time
        assert abs(value - 2e12 * 5 * 2 / 2.0 / 1e12) < 1e-9   # all ranks' work / max time


def test_single_rank_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.throughput_tflops(1e12, 10, 1, 2.0) == 5.0


# ------------------------------------------------------------------ head split
def _split_worker(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, N, H, d = 2, 5, 8, 3
        # a stand-in "output" whose every element names its (b, n, h, c) position
        full = torch.arange(B * N * H * d, dtype=torch.float32).reshape(B, N, H, d)
        h0, h1 = bench.head_range(H, rank, world)
        local = full[:, :, h0:h1].contiguous() * 1.0   # what this rank's attention produced
        out[rank] = (h0, h1, bool(torch.equal(bench.gather_heads(local, world), full)))
    finally:
        dist.destroy_process_group()


def test_two_rank_head_split_and_gather_order():
    # the head partition covers every head once, in rank order, and the all-gather of the
    # ranks' outputs rebuilds the full [B, N, H, d] tensor on every rank
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_split_worker, args=(2, port, out), nprocs=2, join=True,
                       start_method="spawn")
    assert [out[r][:2] for r in range(2)] == [(0, 4), (4, 8)]
    assert out[0][2] and out[1][2]


def test_head_range_rejects_uneven_splits():
    import pytest
    assert bench.head_range(32, 7, 8) == (28, 32)
    with pytest.raises(ValueError):
        bench.head_range(32, 0, 3)
