"""The bench's N-GPU plumbing, run as two gloo ranks on the CPU.

bench.py --gpus N runs one independent replica of the step per GPU (the path
has no exchange step): the only cross-rank operations are a barrier around
the timed region and a max over ranks of the measured times, and the
reference arm runs on rank 0 alone. These tests run that plumbing with
world_size 2 over gloo (no GPU), each rank as its own process.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    bench.dist_init(w, backend="gloo")
    try:
        bench.barrier(w)
        # each rank reports its own time; everyone gets the slowest one
        mx = bench.max_over_ranks(10.0 + rank, w, torch.device("cpu"))
        bench.barrier(w)
        # the reference arm is rank 0's alone: other ranks return at once
        if rank != 0:
            assert bench.reference_arm(None) is None
        with open(os.path.join(out_dir, "rank%d.txt" % rank), "w") as f:
            f.write(repr(mx))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_barrier_and_max_over_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.spawn(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    got = [float(open(tmp_path / ("rank%d.txt" % r)).read()) for r in range(world)]
    assert got == [11.0, 11.0]


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    bench.barrier(1)  # no-op without a process group
    assert not torch.distributed.is_initialized()


def test_weak_scaling_counts_all_ranks_work():
    import bench
    # N replicas each process the same work; the job's value is all ranks'
    # work over the slowest rank's time
    assert bench.weak_scaling_value(2.0e12, 0.5e-3, 1) == pytest.approx(4.0e15)
    assert bench.weak_scaling_value(2.0e12, 0.5e-3, 8) == pytest.approx(8 * 4.0e15)
