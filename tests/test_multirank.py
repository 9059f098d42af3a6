"""The N > 1 path of bench.py (independent replicas, one per GPU), on CPU with
two gloo ranks: every multi-GPU time is the maximum over ranks, and the job's
throughput counts every replica's tokens."""
import datetime
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [1.5, 2.25][rank]          # the second replica is slower
        out[rank] = bench.max_over_ranks(local_ms, "cpu")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
    assert dict(out) == {0: 2.25, 1: 2.25}


def test_single_process_is_a_no_op_and_throughput_counts_all_replicas():
    assert bench.max_over_ranks(3.0, "cpu") == 3.0
    assert bench.job_throughput(2, 1_048_576, 2.0) == 2 * 1_048_576 / 2e-3


def _rank_leaves(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    out[(rank, 0)] = bench.max_over_ranks(1.0 + rank, "cpu")   # step 1: both replicas report
    if rank == 1:
        return                                                  # replica 1 fails between steps and exits
    try:
        bench.max_over_ranks(1.0, "cpu")                        # step 2: the peer is gone
        out[(rank, 1)] = "completed"
    except Exception:
        out[(rank, 1)] = "error"
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_a_replica_that_leaves_between_steps_ends_the_next_timing_with_an_error():
    """A rank that drops out between steps must not hang the others: the next
    max-over-ranks reduction raises (peer closed or the short group timeout)."""
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_leaves, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[(0, 0)] == 2.0 and out[(1, 0)] == 2.0
    assert out[(0, 1)] == "error"
