"""Multi-process host logic of the benchmark at world size 2 over gloo (CPU):
row shards of one batch, whole-job throughput from the slowest rank, the
max-over-ranks reduction, and that reduction ending with an error when a
rank has left.  The quantizer itself has no data-path collective: every rank
works on its own rows."""
import datetime
import os
import socket
import time

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


def _worker_one_leaves(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        # Leaves between steps, with no collective of its own in flight.
        out[1] = "left"
        os._exit(0)
    t0 = time.monotonic()
    try:
        bench.max_over_ranks(1.0)
        out[0] = ("returned", time.monotonic() - t0)
    except Exception as e:                     # the expected outcome
        out[0] = ("raised", time.monotonic() - t0, type(e).__name__)
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


@pytest.mark.timeout(180)
def test_a_rank_that_leaves_ends_the_others_reduction_with_an_error():
    """The max-over-ranks reduction that closes every timed region must not
    wait for good on a rank that has gone: with a short process-group
    timeout the remaining rank gets an error, well inside a minute."""
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    mp.start_processes(_worker_one_leaves, args=(world, _free_port(), out), nprocs=world,
                       join=True, start_method="spawn")
    assert out[1] == "left"
    assert out[0][0] == "raised", out[0]
    assert out[0][1] < 60.0
