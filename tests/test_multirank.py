"""Multi-process host logic of the benchmark at world size 2 over gloo (CPU):
row shards of one batch, whole-job throughput from the slowest rank, and the
max-over-ranks reduction.  The quantizer itself has no data-path collective:
every rank works on its own rows."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads as w


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, lr = bench.dist_env()
        assert (ws, r, lr) == (world, rank, rank)
        rows = 2 * w.ROW_CHUNK
        row0 = bench.shard_row0(rank, rows)
        case = w.make_case("tiny", M=rows, row0=row0)
        # each rank's "time": the slowest one decides the job's time
        ms = 10.0 + 5.0 * rank
        ms_max = bench.max_over_ranks(ms)
        out[rank] = (row0, ms_max, case.x_bits()[:3].copy())
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_rows_and_reduce_time():
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0][0] == 0 and out[1][0] == 2 * w.ROW_CHUNK
    assert out[0][1] == out[1][1] == 15.0
    # rank 1's rows are rows [2 chunks, ...) of the same synthetic batch
    big = w.make_case("tiny", M=4 * w.ROW_CHUNK)
    assert np.array_equal(out[1][2], big.x_bits()[2 * w.ROW_CHUNK:2 * w.ROW_CHUNK + 3])
    assert np.array_equal(out[0][2], big.x_bits()[:3])


def test_aggregate_throughput_counts_every_rank():
    b = w.algorithmic_bytes(16384, 12288)
    one = bench.aggregate_gbs(b, 1, 10, 1.0)
    eight = bench.aggregate_gbs(b, 8, 10, 1.0)
    assert eight == pytest.approx(8 * one)
    assert one == pytest.approx(b * 10 / 1e-3 / 1e9)


def test_single_process_needs_no_process_group():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.5) == 3.5
