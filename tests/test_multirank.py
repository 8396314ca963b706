"""The benchmark's multi-rank plumbing on CPU: two gloo ranks (one process each, as
torchrun would start them) go through bench.py's rendezvous, barrier and max-over-ranks
reduction, which the N-GPU timing uses (each rank times its own replica of the step; the
job's time is the slowest rank's)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    r, w, local = bench.dist_setup(world)
    assert (r, w, local) == (rank, world, rank)
    bench.barrier(w)
    # each rank reports a different time; every rank must see the slowest one
    t = bench.max_over_ranks(10.0 + 5.0 * rank, w, "cpu")
    bench.barrier(w)
    out[rank] = t
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_take_the_max_time():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    bench.barrier(1)
